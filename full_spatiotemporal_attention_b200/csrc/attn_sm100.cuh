// Flash-style attention forward on B200 tensor cores (tcgen05 + TMEM + TMA).
//
//   O = softmax(scale * Q~ K~^T) V over the keys of the query's segment,
//
// where Q~ is Q turned by 3D RoPE inside the kernel (right after its tile
// lands in shared memory) and K~ is the pre-rotated key tensor.  Segments:
// full 3D attention and joint video+text attention use one segment of N
// tokens (handbook "How attention sees time": every token together); the
// spatial pass of factorised attention uses T' segments of H'W' tokens (one
// per frame); local 3D windows use one segment per window, rows gathered token
// by token; text cross-attention ("04 HunyuanVideo and Wan", section 3.1) uses
// one segment of video queries over a separate key/value tensor (the text
// tokens), with no rotation.  The score matrix is never materialised (online
// softmax).
//
// CTA = one (batch*head, segment, NQ x 128 query rows) work tile (KCfg):
//   NQ = 2 (one CTA per SM)      NQ = 1 (two CTAs per SM, short key loops)
//   warps 0-3  softmax group 0   warps 0-3  softmax group 0
//   warps 4-7  softmax group 1   warp  4    MMA issuer, TMEM owner
//   warp  8    MMA issuer        warp  5    TMA loader
//   warp  9    TMA loader        warps 6-7  gathering loaders (windows)
//   warps 10-11 gathering loaders (windows)
// A softmax thread owns one query row (= TMEM lane).
//
// Work units (1-D grid): units below n_whole each cover one NQ x 128-row tile
// over all keys of its segment.  When the last wave would leave SMs idle, its tiles
// are instead covered by two units each, one per half of the key tiles; each
// half writes its normalised fp32 output with its row maximum and sum to the
// workspace, and the second half to finish (a per-tile counter) merges the
// two and writes O.
//
// TMEM (256 NQ columns x 128 lanes, fp32): S_g at 128 g, O_g at 128 (NQ + g);
// P (bf16 pairs) overwrites the first 64 columns of its S.  With NQ = 2 the
// MMA issuer ping-pongs the two query tiles so that one tile's softmax
// overlaps the other tile's QK^T and PV products; with NQ = 1 the two CTAs of
// an SM interleave on its tensor core in the same way, and one CTA's
// prologue and epilogue overlap the other's main loop.  A softmax group
// publishes the P of the first 64 keys of a tile before it computes the rest,
// so that the PV product of those keys runs while it does: a group's next
// scores wait for its own softmax, its PV product and its QK^T product in
// turn, and this takes the first half of the PV product off that chain.  Q, K, V tiles are
// 128 rows x 128 bf16, loaded by TMA as two 64-column boxes with the 128-byte
// swizzle.
#pragma once

#include <type_traits>

#include "ptx.cuh"
#include "rope.cuh"

namespace va3d {
namespace fa {

constexpr int BM = 128;                    // query rows per tile
constexpr int BN = 128;                    // keys per tile
constexpr int HD = 128;                    // head dim
constexpr int kTileBytes = BM * HD * 2;    // 32 KB
constexpr int kHalfBytes = kTileBytes / 2; // one 64-column box: 128 rows x 128 B

enum Bar {
    B_QFULL = 0,
    B_QREADY0, B_QREADY1,
    B_KFULL0, B_KFULL1,
    B_KEMPTY0, B_KEMPTY1,
    B_VFULL0, B_VFULL1,
    B_VEMPTY0, B_VEMPTY1,
    B_SFULL0, B_SFULL1,
    B_PFULL0, B_PFULL1,
    B_PHALF0, B_PHALF1,       // the first 64 keys' P of tile g is in TMEM
    B_OFULL,
    B_DRAIN,
    B_EPI,        // split units: every softmax thread stored its partial
    B_EPI_GO,     // split units: the merge decision is published
    NUM_BARS
};

// Configuration by NQ, the query tiles a CTA holds:
//  NQ = 2: two softmax warpgroups ping-pong on one tensor core, a 2-stage
//          K/V ring, one CTA per SM (long key sequences);
//  NQ = 1: one softmax warpgroup and one K/V stage per CTA, two CTAs per SM
//          that interleave on the tensor core, so that one CTA's prologue and
//          epilogue overlap the other's main loop (short key sequences).
// Warps 0 .. 4NQ-1 are the softmax groups; warp 4NQ issues MMAs and owns
// TMEM, warp 4NQ+1 loads tiles, warps 4NQ+2 and 4NQ+3 gather (windows).
template <int NQ>
struct KCfg {
    static constexpr int kStages = NQ == 2 ? 2 : 1;          // K and V ring depth
    static constexpr int kThreads = 128 * (NQ + 1);
    static constexpr int kMinBlocks = NQ == 2 ? 1 : 2;       // CTAs per SM
    static constexpr int kLaunchRegs = NQ == 2 ? 168 : 128;  // per thread at launch
    // setmaxnreg split (multiples of 8): NQ * 128 * softmax + 128 * producer
    // must fit kThreads * kLaunchRegs.
    static constexpr int kSoftmaxRegs = NQ == 2 ? 216 : 208;
    static constexpr int kProducerRegs = NQ == 2 ? 72 : 48;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + NQ * kTileBytes;
    static constexpr int OFF_V = OFF_K + kStages * kTileBytes;
    static constexpr int OFF_BAR = OFF_V + kStages * kTileBytes;
    static constexpr int OFF_TMEM_SLOT = OFF_BAR + NUM_BARS * 8;
    static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 8;
    static constexpr int OFF_MERGE = OFF_ABORT + 8;   // int: this unit merges the two halves
    static constexpr int kSmemBytes = OFF_MERGE + 8 + 1024;   // slack to align the base
    static constexpr uint32_t kTmemCols = 256 * NQ;   // S_g at 128 g, O_g at 128 (NQ + g)
    static constexpr int kProdWarp = 4 * NQ;
    static_assert(NQ * 128 * kSoftmaxRegs + 128 * kProducerRegs <= kThreads * kLaunchRegs,
                  "register split exceeds the launch allocation");
};

// Lazy rescaling: a row keeps its running maximum (log2 units) until a new
// score exceeds it by more than this; P values then stay below 2^8.
constexpr float kRescaleThreshold = 8.0f;

// Every kPolyEvery-th pair of scores takes the polynomial exp2 (FMA pipe).
constexpr int kPolyEvery = 4;

struct AttnArgs {
    int N;             // query tokens per (batch, head) sequence
    int seg_len;       // query tokens per segment (N, or H'W' for the spatial pass)
    int kv_len;        // keys per segment (seg_len for self-attention; segment s's
                       // keys are rows [s * kv_len, (s + 1) * kv_len) of K and V)
    int q_blocks;      // 256-row query blocks per segment
    int n_seg;         // segments per sequence
    int n_whole;       // units covering a whole tile; the rest are half-key units
    float *part_o;     // [split tiles][2][256][128] normalised partial outputs
    float2 *part_ml;   // [split tiles][2][256] (row maximum in log2 units, row sum)
    int *part_count;   // [split tiles] halves finished
    float scale_log2;  // softmax scale * log2(e)
    int rope_q;        // 1: rotate Q tiles by 3D RoPE (hardware sine and cosine)
    __nv_bfloat16 *o;
    float *lse;        // may be null
    RopeParams rp;
    // Local 3D windows (win != 0): segment s is window s of the grid in
    // (t, h, w) raster order of windows, its rows the window's tokens in
    // (dt, dh, dw) raster order; O and LSE rows are written back to the
    // tokens' natural positions.  win == 2 (window width a multiple of 8 that
    // divides 128): a tile's rows arrive as runs of win_w consecutive tokens,
    // one TMA box each.  win == 1: rows are gathered token by token from the
    // natural-order tensors below.
    int win;
    int win_t, win_h, win_w;   // window size
    int nwin_h, nwin_w;        // windows along h and w
    const __nv_bfloat16 *gq, *gk, *gv;
    // Ring merge (merge != 0, whole units only): this call is one key block
    // of a ring; its normalised output and LSE are merged by log-sum-exp
    // weights into the fp32 accumulator acc [rows, 128] and lse_out (natural
    // log); merge == 1 starts them (first block), merge == 2 folds in lse_in.
    // o, if set, receives the merged output as bf16.
    int merge;
    float *acc;
    const float *lse_in;
    float *lse_out;
    // O written by TMA store from the group's Q tile: 1 = one box of 128
    // rows per half (map: [n_seg * BH] segments of seg_len rows), 2 = one box
    // per window run (map: [BH, N] rows, boxes of win_w rows); 0 = row stores
    int o_tma;
};

// Natural token index of row `local` of window `seg`.
__device__ __forceinline__ int window_token(const AttnArgs &a, int seg, int local) {
    const int dw = local % a.win_w;
    const int rest = local / a.win_w;
    const int dh = rest % a.win_h;
    const int dt = rest / a.win_h;
    const int cw = seg % a.nwin_w;
    const int rest2 = seg / a.nwin_w;
    const int ch = rest2 % a.nwin_h;
    const int ct = rest2 / a.nwin_h;
    return ((ct * a.win_t + dt) * a.rp.H + ch * a.win_h + dh) * a.rp.W + cw * a.win_w + dw;
}

__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) {
    // K-major, 128 B swizzle: 8-row groups 1024 B apart; the leading offset
    // is unused for this layout (encoded as 16 B).
    return smem_desc_sw128(saddr, 16, 1024);
}

__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr) {
    // MN-major, 128 B swizzle: the two 64-element column blocks are one box
    // (16 KB) apart; 8-row groups along K are 1024 B apart.
    return smem_desc_sw128(saddr, kHalfBytes, 1024);
}

// Turn row `r` of a swizzled 128x128 Q tile in shared memory by 3D RoPE.
// All 64 (cos, sin) pairs of the row are formed first, from the hardware sine
// and cosine of pos * inv_freq (absolute error ~1e-5 at the largest angles of
// the pages' grids, far below the bf16 rounding of the turned values; 3.4k
// cycles per tile against 9k for 64 angle-table loads per row), then the row
// is rotated in place.
__device__ __forceinline__ void rope_q_row(uint8_t *tile, int r, int n, const AttnArgs &a) {
    const RopeParams &rp = a.rp;
    if (n >= rp.n_video) return;   // text token or a padding row past N
    const int t = n / rp.HW;
    const int rem = n - t * rp.HW;
    const int h = rem / rp.W;
    const int w = rem - h * rp.W;
    float2 cs[64];
#pragma unroll
    for (int p = 0; p < 64; ++p) {
        const float ang = static_cast<float>(pair_pos(rp, p, t, h, w)) * rp.inv_freq[p];
        __sincosf(ang, &cs[p].y, &cs[p].x);
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4 *ptr = reinterpret_cast<uint4 *>(tile + half * kHalfBytes + r * 128 +
                                                   ((c ^ (r & 7)) << 4));
            uint4 v = *ptr;
            const int p0 = half * 32 + c * 4;
            v.x = rotate_pair(v.x, cs[p0 + 0]);
            v.y = rotate_pair(v.y, cs[p0 + 1]);
            v.z = rotate_pair(v.z, cs[p0 + 2]);
            v.w = rotate_pair(v.w, cs[p0 + 3]);
            *ptr = v;
        }
    }
}

template <int NQ>
__global__ void __launch_bounds__(KCfg<NQ>::kThreads, KCfg<NQ>::kMinBlocks)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                const __grid_constant__ AttnArgs a) {
    using C = KCfg<NQ>;
    constexpr int kStages = C::kStages;
    constexpr int OFF_Q = C::OFF_Q, OFF_K = C::OFF_K, OFF_V = C::OFF_V;
    constexpr int OFF_TMEM_SLOT = C::OFF_TMEM_SLOT, OFF_MERGE = C::OFF_MERGE;
    constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 128 * NQ, COL_O1 = 128 * NQ + 128;
    constexpr int kMma = C::kProdWarp, kLoad = C::kProdWarp + 1, kGather = C::kProdWarp + 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const uint32_t sbase = smem_u32(smem);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_ABORT);
    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8 * i; };
    // tile j of the K/V stream: stage and phase of the ring
    auto stg = [](int j) { return j % kStages; };
    auto phs = [](int j) -> uint32_t { return static_cast<uint32_t>((j / kStages) & 1); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // unit -> tile and key-tile range [j0, j1)
    const int unit = blockIdx.x;
    const bool split = unit >= a.n_whole;
    const int split_idx = split ? (unit - a.n_whole) >> 1 : 0;
    const int part = split ? (unit - a.n_whole) & 1 : 0;
    const int tile = split ? a.n_whole + split_idx : unit;
    const int qb = tile % a.q_blocks;
    const int seg = (tile / a.q_blocks) % a.n_seg;
    const int bh = tile / (a.q_blocks * a.n_seg);
    const int seg_start = seg * a.seg_len;
    const int seg_end = seg_start + a.seg_len;
    const int q0 = seg_start + qb * (NQ * BM);
    const int kv_start = seg * a.kv_len;
    const int n_kv_all = (a.kv_len + BN - 1) / BN;
    const int kv_last_valid = a.kv_len - (n_kv_all - 1) * BN;
    const int j0 = split && part ? n_kv_all / 2 : 0;
    const int j1 = split && !part ? n_kv_all / 2 : n_kv_all;
    const int n_kv = j1 - j0;   // key tiles of this unit; local step jj = j - j0
    // Two query tiles, unless the second lies wholly past the segment (the
    // last block of a segment shorter than it): then only tile 0 is computed
    // and the second softmax group idles.  Split units keep both (their merge
    // counts the rows of both tiles).
    const bool two = NQ == 2 && (split || q0 + BM < seg_end);

    if (threadIdx.x == 0) {
        mbar_init(bar(B_QFULL), 1);
        mbar_init(bar(B_QREADY0), BM);
        mbar_init(bar(B_QREADY1), BM);
        // full barriers: one TMA arrival with its byte count, or one arrival
        // per gathering thread in window mode
        const uint32_t full_count = a.win == 1 ? 64u : 1u;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(B_KFULL0 + s), full_count);
            mbar_init(bar(B_KEMPTY0 + s), 1);
            mbar_init(bar(B_VFULL0 + s), full_count);
            mbar_init(bar(B_VEMPTY0 + s), 1);
        }
        mbar_init(bar(B_SFULL0), 1);
        mbar_init(bar(B_SFULL1), 1);
        mbar_init(bar(B_PFULL0), BM);
        mbar_init(bar(B_PFULL1), BM);
        mbar_init(bar(B_PHALF0), BM);
        mbar_init(bar(B_PHALF1), BM);
        mbar_init(bar(B_OFULL), 1);
        mbar_init(bar(B_DRAIN), 1);
        mbar_init(bar(B_EPI), NQ * BM);
        mbar_init(bar(B_EPI_GO), 1);
        *abort_flag = 0;
        mbar_init_fence();
        fence_proxy_async_smem();
    }
    if (warp == kMma) tmem_alloc(sbase + OFF_TMEM_SLOT, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + OFF_TMEM_SLOT);
    // Each role runs inside the branch that set its register budget (the new
    // budget applies to the code that instruction dominates).
    if (warp >= kMma) {
    regs_lower<C::kProducerRegs>();
    if (warp >= kGather) {
        // ------------------------------------------- gathering loader (windows)
        // 64 threads copy the K and V rows of each key tile token by token
        // (16-byte cp.async into the same swizzled layout TMA produces), two
        // tiles in flight; after its copies land a thread fences them for the
        // tensor core's proxy and arrives on the tile's full barrier.
        if (a.win == 1) {
            const int lt = threadIdx.x - kGather * 32;   // 0..63
            auto gather = [&](const __nv_bfloat16 *src, uint32_t dst, int j) {
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int i = lt * 2 + h2;                 // row of the tile
                    const int local = (j0 + j) * BN + i;       // row of the window
                    const uint32_t row = dst + i * 128;
                    if (local < a.kv_len) {
                        const __nv_bfloat16 *g =
                            src + (static_cast<size_t>(bh) * a.N + window_token(a, seg, local)) * HD;
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            cp_async16(row + (c >> 3) * kHalfBytes + (((c & 7) ^ (i & 7)) << 4), g + c * 8);
                    } else {
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            st_shared_zero16(row + (c >> 3) * kHalfBytes + (((c & 7) ^ (i & 7)) << 4));
                    }
                }
            };
            // Commit groups go K(0), V(0), K(1), V(1), ...  Step j publishes
            // K(j-1) and V(j-1) as soon as each has landed and issues K(j) and
            // V(j) once their stages are released, so up to one K and one V
            // tile are in flight besides the ones being published.
            bool ok = true;
            for (int j = 0; j <= n_kv && ok; ++j) {
                const int s = stg(j);
                const uint32_t ph = phs(j);
                if (j >= 1) {
                    cp_async_wait<1>();                  // K(j-1); V(j-1) may be pending
                    fence_proxy_async_smem();
                    mbar_arrive(bar(B_KFULL0 + stg(j - 1)));
                }
                if (j < n_kv) {
                    if (j >= kStages &&
                        !(ok = mbar_wait(bar(B_KEMPTY0 + s), ph ^ 1, abort_flag, VA3D_DEVERR_TIMEOUT_LOAD)))
                        break;
                    gather(a.gk, sbase + OFF_K + s * kTileBytes, j);
                    cp_async_commit();
                }
                if (j >= 1) {
                    if (j < n_kv)
                        cp_async_wait<1>();              // V(j-1); K(j) may be pending
                    else
                        cp_async_wait<0>();
                    fence_proxy_async_smem();
                    mbar_arrive(bar(B_VFULL0 + stg(j - 1)));
                }
                if (j < n_kv) {
                    if (j >= kStages &&
                        !(ok = mbar_wait(bar(B_VEMPTY0 + s), ph ^ 1, abort_flag, VA3D_DEVERR_TIMEOUT_LOAD)))
                        break;
                    gather(a.gv, sbase + OFF_V + s * kTileBytes, j);
                    cp_async_commit();
                }
            }
            cp_async_wait<0>();
            if (ok) {
                // every released stage was consumed; wait for the last tiles'
                // releases so no arrival lands after the CTA exits
                const int first = n_kv > kStages ? n_kv - kStages : 0;
                for (int j = first; j < n_kv && ok; ++j)
                    ok = mbar_wait(bar(B_KEMPTY0 + stg(j)), phs(j), abort_flag,
                                   VA3D_DEVERR_TIMEOUT_LOAD) &&
                         mbar_wait(bar(B_VEMPTY0 + stg(j)), phs(j), abort_flag,
                                   VA3D_DEVERR_TIMEOUT_LOAD);
            }
        }
    } else if (warp == kLoad) {
        // ------------------------------------------------------------ loader
        if (a.win == 2) {
            // -------------------------------------------- window runs loader
            // A tile's rows arrive as runs of win_w consecutive tokens, one box
            // of the win_w-row maps each; lane u issues run u of every tile.
            // Runs past the window repeat its last run (those rows are masked
            // as keys and not stored as queries).
            const int runs = BM / a.win_w;
            const int n_runs = a.seg_len / a.win_w;
            const int origin = window_token(a, seg, 0);
            auto load_runs = [&](const CUtensorMap *map, uint32_t dst, uint32_t fbar, int local0) {
                if (lane < runs) {
                    const int run = min(local0 / a.win_w + lane, n_runs - 1);
                    const int dt = run / a.win_h, dh = run - dt * a.win_h;
                    const int row = origin + dt * a.rp.HW + dh * a.rp.W;
                    for (int hf = 0; hf < 2; ++hf)
                        tma_load_3d(dst + hf * kHalfBytes + lane * a.win_w * 128, map, fbar, hf * 64, row, bh);
                }
            };
            if (lane == 0) {
                tma_prefetch_desc(&tmQ);
                tma_prefetch_desc(&tmK);
                tma_prefetch_desc(&tmV);
                mbar_arrive_expect_tx(bar(B_QFULL), NQ * kTileBytes);
            }
            __syncwarp();
            for (int i = 0; i < NQ; ++i)
                load_runs(&tmQ, sbase + OFF_Q + i * kTileBytes, bar(B_QFULL), q0 - seg_start + i * BM);
            int k_issued = 0, v_issued = 0;
            bool ok = true;
            for (int j = 0; j < n_kv; ++j) {
                const int s = stg(j);
                const uint32_t ph = phs(j);
                if (j >= kStages &&
                    !(ok = __all_sync(0xffffffffu, mbar_wait(bar(B_KEMPTY0 + s), ph ^ 1, abort_flag,
                                                             VA3D_DEVERR_TIMEOUT_LOAD))))
                    break;
                if (lane == 0) mbar_arrive_expect_tx(bar(B_KFULL0 + s), kTileBytes);
                __syncwarp();
                load_runs(&tmK, sbase + OFF_K + s * kTileBytes, bar(B_KFULL0 + s), (j0 + j) * BN);
                k_issued = j + 1;
                if (j >= kStages &&
                    !(ok = __all_sync(0xffffffffu, mbar_wait(bar(B_VEMPTY0 + s), ph ^ 1, abort_flag,
                                                             VA3D_DEVERR_TIMEOUT_LOAD))))
                    break;
                if (lane == 0) mbar_arrive_expect_tx(bar(B_VFULL0 + s), kTileBytes);
                __syncwarp();
                load_runs(&tmV, sbase + OFF_V + s * kTileBytes, bar(B_VFULL0 + s), (j0 + j) * BN);
                v_issued = j + 1;
            }
            const int k_first = k_issued > kStages ? k_issued - kStages : 0;
            const int v_first = v_issued > kStages ? v_issued - kStages : 0;
            if (ok) {
                for (int j = k_first; j < k_issued && ok; ++j)
                    ok = __all_sync(0xffffffffu, mbar_wait(bar(B_KEMPTY0 + stg(j)), phs(j), abort_flag,
                                                           VA3D_DEVERR_TIMEOUT_LOAD));
                for (int j = v_first; j < v_issued && ok; ++j)
                    ok = __all_sync(0xffffffffu, mbar_wait(bar(B_VEMPTY0 + stg(j)), phs(j), abort_flag,
                                                           VA3D_DEVERR_TIMEOUT_LOAD));
            }
            if (!ok) {
                // Let the copies already in flight land before the CTA exits.
                mbar_wait_drain(bar(B_QFULL), 0);
                for (int j = k_first; j < k_issued; ++j)
                    mbar_wait_drain(bar(B_KFULL0 + stg(j)), phs(j));
                for (int j = v_first; j < v_issued; ++j)
                    mbar_wait_drain(bar(B_VFULL0 + stg(j)), phs(j));
            }
        } else if (lane == 0 && !a.win) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(bar(B_QFULL), NQ * kTileBytes);
            for (int i = 0; i < NQ; ++i)
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_3d(sbase + OFF_Q + i * kTileBytes + hf * kHalfBytes, &tmQ,
                                bar(B_QFULL), hf * 64, q0 + i * BM, bh);
            // Tile j goes to stage stg(j) with phase phs(j); only the last
            // kStages issued tiles can still be in flight or unreleased.
            int k_issued = 0, v_issued = 0;
            bool ok = true;
            for (int j = 0; j < n_kv; ++j) {
                const int s = stg(j);
                const uint32_t ph = phs(j);
                const int kv0 = kv_start + (j0 + j) * BN;
                if (j >= kStages &&
                    !(ok = mbar_wait(bar(B_KEMPTY0 + s), ph ^ 1, abort_flag, VA3D_DEVERR_TIMEOUT_LOAD)))
                    break;
                mbar_arrive_expect_tx(bar(B_KFULL0 + s), kTileBytes);
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_3d(sbase + OFF_K + s * kTileBytes + hf * kHalfBytes, &tmK,
                                bar(B_KFULL0 + s), hf * 64, kv0, bh);
                k_issued = j + 1;
                if (j >= kStages &&
                    !(ok = mbar_wait(bar(B_VEMPTY0 + s), ph ^ 1, abort_flag, VA3D_DEVERR_TIMEOUT_LOAD)))
                    break;
                mbar_arrive_expect_tx(bar(B_VFULL0 + s), kTileBytes);
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_3d(sbase + OFF_V + s * kTileBytes + hf * kHalfBytes, &tmV,
                                bar(B_VFULL0 + s), hf * 64, kv0, bh);
                v_issued = j + 1;
            }
            const int k_first = k_issued > kStages ? k_issued - kStages : 0;
            const int v_first = v_issued > kStages ? v_issued - kStages : 0;
            if (ok) {
                // Producer tail: wait until the last tile of each stage has been
                // released, so no barrier arrival can land after the CTA exits.
                for (int j = k_first; j < k_issued && ok; ++j)
                    ok = mbar_wait(bar(B_KEMPTY0 + stg(j)), phs(j), abort_flag,
                                   VA3D_DEVERR_TIMEOUT_LOAD);
                for (int j = v_first; j < v_issued && ok; ++j)
                    ok = mbar_wait(bar(B_VEMPTY0 + stg(j)), phs(j), abort_flag,
                                   VA3D_DEVERR_TIMEOUT_LOAD);
            }
            if (!ok) {
                // Let the copies already in flight land before the CTA exits.
                mbar_wait_drain(bar(B_QFULL), 0);
                for (int j = k_first; j < k_issued; ++j)
                    mbar_wait_drain(bar(B_KFULL0 + stg(j)), phs(j));
                for (int j = v_first; j < v_issued; ++j)
                    mbar_wait_drain(bar(B_VFULL0 + stg(j)), phs(j));
            }
        }
    } else if (warp == kMma) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescQK = idesc_bf16_f32(BM, BN, 0);
            constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, HD, 1);

            auto issue_s = [&](int i, int s) {
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + COL_S0 + i * (COL_S1 - COL_S0), desc_kmajor(sbase + OFF_Q + i * kTileBytes + off),
                           desc_kmajor(sbase + OFF_K + s * kTileBytes + off), kIdescQK, kk > 0);
                }
            };
            auto issue_pv = [&](int i, int s, bool acc, int k_lo, int k_hi) {
#pragma unroll
                for (int kk = k_lo; kk < k_hi; ++kk) {
                    mma_ts(tmem + COL_O0 + i * (COL_O1 - COL_O0), tmem + COL_S0 + i * (COL_S1 - COL_S0) + kk * 8,
                           desc_mnmajor(sbase + OFF_V + s * kTileBytes + kk * 2048), kIdescPV,
                           (acc || kk > 0) ? 1u : 0u);
                }
            };

            bool ok = mbar_wait(bar(B_QREADY0), 0, abort_flag, VA3D_DEVERR_TIMEOUT_MMA) &&
                      (!two || mbar_wait(bar(B_QREADY1), 0, abort_flag, VA3D_DEVERR_TIMEOUT_MMA)) &&
                      mbar_wait(bar(B_KFULL0), 0, abort_flag, VA3D_DEVERR_TIMEOUT_MMA);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                mma_commit(bar(B_SFULL0));
                if (two) {
                    issue_s(1, 0);
                    mma_commit(bar(B_SFULL1));
                }
                mma_commit(bar(B_KEMPTY0));
            }
            for (int j = 0; j < n_kv && ok; ++j) {
                const int s = stg(j);
                const uint32_t ph = phs(j);
                const bool more = j + 1 < n_kv;
                const int s2 = stg(j + 1);
                const uint32_t ph2 = phs(j + 1);
                ok = mbar_wait(bar(B_VFULL0 + s), ph, abort_flag, VA3D_DEVERR_TIMEOUT_MMA) &&
                     mbar_wait(bar(B_PHALF0), j & 1, abort_flag, VA3D_DEVERR_TIMEOUT_MMA);
                if (!ok) break;
                tc_fence_after();
                issue_pv(0, s, j > 0, 0, 4);
                ok = mbar_wait(bar(B_PFULL0), j & 1, abort_flag, VA3D_DEVERR_TIMEOUT_MMA);
                if (!ok) break;
                tc_fence_after();
                issue_pv(0, s, true, 4, 8);
                // one query tile: V's stage is free after this product.  (Its
                // release must not wait for the next QK^T: with one stage the
                // gathering loader publishes that K tile only after refilling V.)
                if (!two) mma_commit(bar(B_VEMPTY0 + s));
                if (more) {
                    ok = mbar_wait(bar(B_KFULL0 + s2), ph2, abort_flag, VA3D_DEVERR_TIMEOUT_MMA);
                    if (!ok) break;
                    tc_fence_after();
                    issue_s(0, s2);
                    mma_commit(bar(B_SFULL0));
                }
                if (two) {
                    ok = mbar_wait(bar(B_PHALF1), j & 1, abort_flag, VA3D_DEVERR_TIMEOUT_MMA);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(1, s, j > 0, 0, 4);
                    ok = mbar_wait(bar(B_PFULL1), j & 1, abort_flag, VA3D_DEVERR_TIMEOUT_MMA);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(1, s, true, 4, 8);
                    mma_commit(bar(B_VEMPTY0 + s));
                }
                if (more) {
                    if (two) {
                        issue_s(1, s2);
                        mma_commit(bar(B_SFULL1));
                    }
                    mma_commit(bar(B_KEMPTY0 + s2));
                }
            }
            if (ok) {
                mma_commit(bar(B_OFULL));
            } else {
                // Wait for the products already issued before TMEM is freed.
                mma_commit(bar(B_DRAIN));
                mbar_wait_drain(bar(B_DRAIN), 0);
            }
        }
    }
    } else if (warp < 4 || two) {
        regs_raise<C::kSoftmaxRegs>();
        // ---------------------------------------------------------- softmax
        const int g = warp >> 2;                  // query tile of this group
        const int r = ((warp & 3) << 5) + lane;   // row in the tile = TMEM lane
        const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) << 5) << 16;
        const uint32_t taS = tmem + lane_addr + (g ? COL_S1 : COL_S0);
        const uint32_t taO = tmem + lane_addr + (g ? COL_O1 : COL_O0);
        const int n = q0 + g * BM + r;            // token index of this row

        // natural token index of this row (differs from n only for windows)
        const int n_out = a.win && n < seg_end ? window_token(a, seg, n - seg_start) : n;
        bool ok = true;
        if (a.win == 1) {
            // gather this row of Q itself (256 contiguous bytes) into the
            // swizzled tile; rows past the window are zero
            uint8_t *tile = smem + OFF_Q + g * kTileBytes;
            const bool in = n < seg_end;
            uint4 row[16];
            if (in) {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    a.gq + (static_cast<size_t>(bh) * a.N + n_out) * HD);
#pragma unroll
                for (int c = 0; c < 16; ++c) row[c] = __ldg(src + c);
            } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) row[c] = make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int c = 0; c < 16; ++c)
                *reinterpret_cast<uint4 *>(tile + (c >> 3) * kHalfBytes + r * 128 +
                                           (((c & 7) ^ (r & 7)) << 4)) = row[c];
            if (a.rope_q && in) rope_q_row(tile, r, n_out, a);
            fence_proxy_async_smem();
            mbar_arrive(bar(g ? B_QREADY1 : B_QREADY0));
        } else {
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_QFULL), 0, abort_flag,
                                                   VA3D_DEVERR_TIMEOUT_SOFTMAX));
            if (ok) {
                if (a.rope_q) rope_q_row(smem + OFF_Q + g * kTileBytes, r, n_out, a);
                fence_proxy_async_smem();
                mbar_arrive(bar(g ? B_QREADY1 : B_QREADY0));
            }
        }

        float m_ref = -INFINITY;   // running row maximum, log2 units (scaled)
        float l = 0.0f;            // running row sum of exp2
        for (int j = 0; j < n_kv && ok; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar(g ? B_SFULL1 : B_SFULL0), j & 1,
                                                   abort_flag, VA3D_DEVERR_TIMEOUT_SOFTMAX));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[128];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld32(taS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
            float *s = reinterpret_cast<float *>(sr);
            const bool masked_tile = (j0 + j == n_kv_all - 1) && (kv_last_valid < BN);
            if (masked_tile) {
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (c >= kv_last_valid) s[c] = -INFINITY;
            }
            // row maximum: a tree of three-input max (depth 5)
            float t1[43];
#pragma unroll
            for (int q = 0; q < 42; ++q) t1[q] = fmax3(s[3 * q], s[3 * q + 1], s[3 * q + 2]);
            t1[42] = fmaxf(s[126], s[127]);
            float t2[15];
#pragma unroll
            for (int q = 0; q < 14; ++q) t2[q] = fmax3(t1[3 * q], t1[3 * q + 1], t1[3 * q + 2]);
            t2[14] = t1[42];
            float t3[5];
#pragma unroll
            for (int q = 0; q < 5; ++q) t3[q] = fmax3(t2[3 * q], t2[3 * q + 1], t2[3 * q + 2]);
            const float mx = fmaxf(fmax3(t3[0], t3[1], t3[2]), fmaxf(t3[3], t3[4]));
            const float m_new = fmaxf(m_ref, mx * a.scale_log2);
            float alpha = 1.0f;
            const bool bump = m_new - m_ref > kRescaleThreshold;
            if (bump) {
                alpha = ex2(m_ref - m_new);
                m_ref = m_new;
            }
            // O must be rescaled before the first PV product of this tile
            if (j > 0 && __any_sync(0xffffffffu, bump)) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(taO + 32 * c, ov);
                    tmem_wait_ld();
                    reg_fence32(ov);
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                    tmem_st32(taO + 32 * c, ov);
                }
            }
            // P = 2^(s*scale - m) in pairs; a quarter of the pairs use the FMA-pipe
            // exp2 to offload the MUFU unit (not on the masked tile, whose -inf
            // scores need an exact zero); four independent fp32x2 partial sums.
            const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
            const float2 nm2 = make_float2(-m_ref, -m_ref);
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
            auto exp_store = [&](auto mixed) {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int e = 64 * hf + 2 * c;
                        const float2 x = fma2(make_float2(s[e], s[e + 1]), sc2, nm2);
                        float2 p;
                        if (decltype(mixed)::value && (c % kPolyEvery) == kPolyEvery - 1)
                            p = exp2_poly(x);
                        else
                            p = make_float2(ex2(x.x), ex2(x.y));
                        acc[c & 3] = add2(acc[c & 3], p);
                        pk[c] = pack_bf16x2(p.x, p.y);
                    }
                    tmem_st32(taS + 32 * hf, pk);
                    if (hf == 0) {
                        // the first 64 keys' P: the MMA issuer may start on them
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(bar(g ? B_PHALF1 : B_PHALF0));
                    }
                }
            };
            if (masked_tile)
                exp_store(std::false_type{});
            else
                exp_store(std::true_type{});
            const float2 acc01 = add2(acc[0], acc[1]);
            const float2 acc23 = add2(acc[2], acc[3]);
            const float2 acc_all = add2(acc01, acc23);
            const float rowsum = acc_all.x + acc_all.y;
            l = l * alpha + rowsum;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(g ? B_PFULL1 : B_PFULL0));
        }

        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OFULL), 0, abort_flag,
                                                       VA3D_DEVERR_TIMEOUT_SOFTMAX));
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const bool valid = n < seg_end;
            uint4 *dst = reinterpret_cast<uint4 *>(a.o + (static_cast<size_t>(bh) * a.N + n_out) * HD);
            if (a.merge) {
                // ring block: merge into the accumulator by log-sum-exp weights
                //   l = m + log(e^(l_in - m) + e^(l_blk - m)),
                //   o = (e^(l_in - m) o_in + e^(l_blk - m) o_blk) / (...),
                // in log2 units (m_ref and l give the block's log2-sum-exp)
                const size_t row = static_cast<size_t>(bh) * a.N + n_out;
                const float lb2 = m_ref + log2f(l);
                float wa = 0.0f, wb = 1.0f, lo2 = lb2;
                if (a.merge == 2 && valid) {
                    const float la2 = a.lse_in[row] * 1.4426950408889634f;
                    const float mm = fmaxf(la2, lb2);
                    const float ea = ex2(la2 - mm), eb = ex2(lb2 - mm);
                    const float inv = 1.0f / (ea + eb);
                    wa = ea * inv;
                    wb = eb * inv;
                    lo2 = mm + log2f(ea + eb);
                }
                float4 *accp = reinterpret_cast<float4 *>(a.acc + row * HD);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(taO + 32 * c, ov);
                    tmem_wait_ld();
                    reg_fence32(ov);
                    if (valid) {
                        float x[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(ov[e]) * inv_l * wb;
                        if (a.merge == 2) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const float4 y = accp[c * 8 + e];
                                x[4 * e] += wa * y.x;
                                x[4 * e + 1] += wa * y.y;
                                x[4 * e + 2] += wa * y.z;
                                x[4 * e + 3] += wa * y.w;
                            }
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            accp[c * 8 + e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                        if (a.o != nullptr) {
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                dst[c * 4 + e] = make_uint4(pack_bf16x2(x[8 * e], x[8 * e + 1]),
                                                            pack_bf16x2(x[8 * e + 2], x[8 * e + 3]),
                                                            pack_bf16x2(x[8 * e + 4], x[8 * e + 5]),
                                                            pack_bf16x2(x[8 * e + 6], x[8 * e + 7]));
                        }
                    }
                }
                if (valid) a.lse_out[row] = lo2 * 0.69314718055994531f;
            } else if (!split) {
                // O rows staged in this group's Q tile (its products are all
                // done) for the TMA store below, or written row by row
                uint8_t *stage = smem + OFF_Q + g * kTileBytes;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(taO + 32 * c, ov);
                    tmem_wait_ld();
                    reg_fence32(ov);
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv_l,
                                            __uint_as_float(ov[2 * e + 1]) * inv_l);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint4 w4 = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                        const int cc = c * 4 + e;   // 16-byte chunk of the row
                        if (a.o_tma)
                            *reinterpret_cast<uint4 *>(stage + (cc >> 3) * kHalfBytes + r * 128 +
                                                       (((cc & 7) ^ (r & 7)) << 4)) = w4;
                        else if (valid)
                            dst[cc] = w4;
                    }
                }
                if (a.lse != nullptr && valid)
                    a.lse[static_cast<size_t>(bh) * a.N + n_out] = (m_ref + log2f(l)) * 0.69314718055994531f;
            } else {
                // half of the keys: store the normalised partial and its (max, sum)
                const size_t prow = (static_cast<size_t>(split_idx) * 2 + part) * (2 * BM) + g * BM + r;
                // (the scratch holds 256 rows per half whatever NQ)
                float4 *po = reinterpret_cast<float4 *>(a.part_o + prow * HD);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(taO + 32 * c, ov);
                    tmem_wait_ld();
                    reg_fence32(ov);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        po[c * 8 + e] = make_float4(__uint_as_float(ov[4 * e]) * inv_l,
                                                    __uint_as_float(ov[4 * e + 1]) * inv_l,
                                                    __uint_as_float(ov[4 * e + 2]) * inv_l,
                                                    __uint_as_float(ov[4 * e + 3]) * inv_l);
                }
                a.part_ml[prow] = make_float2(m_ref, l);
                __threadfence();
                mbar_arrive(bar(B_EPI));
                volatile int *merge = reinterpret_cast<volatile int *>(smem + OFF_MERGE);
                if (threadIdx.x == 0) {
                    // all 256 rows of this half are stored and fenced: count it
                    ok = mbar_wait(bar(B_EPI), 0, abort_flag, VA3D_DEVERR_TIMEOUT_SOFTMAX);
                    *merge = ok ? atomicAdd(&a.part_count[split_idx], 1) : 0;
                    __threadfence();
                    mbar_arrive(bar(B_EPI_GO));
                }
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_EPI_GO), 0, abort_flag,
                                                       VA3D_DEVERR_TIMEOUT_SOFTMAX));
                if (ok && *merge == 1) {
                    // the other half finished first: merge both and write O
                    __threadfence();
                    const size_t orow = (static_cast<size_t>(split_idx) * 2 + (1 - part)) * (2 * BM) + g * BM + r;
                    const float2 ml_o = __ldcg(&a.part_ml[orow]);
                    const float m_max = fmaxf(m_ref, ml_o.x);
                    const float w_s = l * ex2(m_ref - m_max);
                    const float w_o = ml_o.y * ex2(ml_o.x - m_max);
                    const float inv_w = 1.0f / (w_s + w_o);
                    const float c_s = w_s * inv_w, c_o = w_o * inv_w;
                    const float4 *pa = reinterpret_cast<const float4 *>(a.part_o + prow * HD);
                    const float4 *pb = reinterpret_cast<const float4 *>(a.part_o + orow * HD);
#pragma unroll 4
                    for (int c = 0; c < 16; ++c) {
                        const float4 x0 = __ldcg(pa + 2 * c), x1 = __ldcg(pa + 2 * c + 1);
                        const float4 y0 = __ldcg(pb + 2 * c), y1 = __ldcg(pb + 2 * c + 1);
                        if (valid)
                            dst[c] = make_uint4(pack_bf16x2(x0.x * c_s + y0.x * c_o, x0.y * c_s + y0.y * c_o),
                                                pack_bf16x2(x0.z * c_s + y0.z * c_o, x0.w * c_s + y0.w * c_o),
                                                pack_bf16x2(x1.x * c_s + y1.x * c_o, x1.y * c_s + y1.y * c_o),
                                                pack_bf16x2(x1.z * c_s + y1.z * c_o, x1.w * c_s + y1.w * c_o));
                    }
                    if (a.lse != nullptr && valid)
                        a.lse[static_cast<size_t>(bh) * a.N + n_out] =
                            (m_max + log2f(w_s + w_o)) * 0.69314718055994531f;
                }
            }
        }
        if (a.o_tma && !split && !a.merge) {
            // every row of the group is staged (or a wait gave up: then no
            // store); the store clips rows past the segment (o_tma == 1: one
            // box of 128 rows per half) or stores only the window's runs
            // (o_tma == 2: one box of win_w rows per run, natural positions).
            // The CTA may leave once the store has read shared memory; its
            // writes complete before the grid does.
            fence_proxy_async_smem();
            const bool all_ok = named_and(1 + g, BM, ok);
            const uint32_t stage = sbase + OFF_Q + g * kTileBytes;
            if (all_ok && (warp & 3) == 0) {
                if (a.o_tma == 1) {
                    if (lane == 0) {
                        for (int hf = 0; hf < 2; ++hf)
                            tma_store_3d(&tmO, stage + hf * kHalfBytes, hf * 64,
                                         q0 - seg_start + g * BM, bh * a.n_seg + seg);
                        bulk_commit_group();
                        bulk_wait_group_read0();
                    }
                } else {
                    const int runs = BM / a.win_w;
                    const int run = (q0 - seg_start + g * BM) / a.win_w + lane;
                    if (lane < runs && run < a.seg_len / a.win_w) {
                        const int dt = run / a.win_h, dh = run - dt * a.win_h;
                        const int row = window_token(a, seg, 0) + dt * a.rp.HW + dh * a.rp.W;
                        for (int hf = 0; hf < 2; ++hf)
                            tma_store_3d(&tmO, stage + hf * kHalfBytes + lane * a.win_w * 128, hf * 64,
                                         row, bh);
                        bulk_commit_group();
                        bulk_wait_group_read0();
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMma) tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace fa
}  // namespace va3d

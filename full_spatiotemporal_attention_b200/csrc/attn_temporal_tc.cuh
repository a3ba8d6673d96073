// Temporal pass of factorised attention on the tensor cores (tcgen05 + TMEM +
// TMA), for T' <= 32 frames (handbook "How attention sees time": at each
// spatial position, attention along time over the T' tokens that share its
// (h, w); token (t, h, w) sits at row t*H'W' + h*W' + w).
//
// Tiles.  A 128-row tile holds P = 128 / R positions, each as R rows (its T'
// frames, then zero rows), R = 8, 16 or 32, the least of them >= T': one 4D
// TMA box (64 dims, R frames, P positions, 1 batch*head) per 64-dim half
// lands them as tile row p*R + frame, with frames past T' and positions past
// H'W' zero-filled by the copy.  S = Q K^T is one 128x128 product per tile;
// the row of position p only uses its own R key columns, and as R divides 32
// the positions of warp w's 32 rows own exactly key columns [32w, 32w + 32):
// a warp reads 32 columns of S instead of 128.
//
// P lives in its own TMEM columns.  Row r's P is zero outside its position's
// block; only the block changes from tile to tile (row r always belongs to
// the same local position), so the region is zeroed once and each tile
// rewrites only the warp's span.  O = P V then runs as one 128x128x128 product
// whose off-block terms are exact zeros, into the columns S occupied.
//
// Raw keys (the usual call): within one position every row has the same
// (h, w), so the h and w rotations of Q and K cancel in q.k and only the t
// range needs turning.  Each thread turns the first ceil16(d_t) dims of its
// row of Q and K in place as fp16; the QK^T k-steps over those dims run as
// fp16 x fp16 products, the rest as bf16 x bf16 on the untouched inputs (exact
// products), all into one fp32 accumulator.  Keys that come rotated: Q is
// turned in full and K converted, both fp16, and all of QK^T runs in fp16.
// If the values written leave fp16's comfortable range, the tile is redone
// with all dims in fp16 under per-tile powers of two.
//
// Roles: two groups of four warps, each running its own tiles (the CTA's
// even and odd tiles) through its own Q/K stage, V stage and TMEM columns, so
// one group's loads and products overlap the other's arithmetic.  Thread 0 of
// a group issues its products and refills its stages: Q/K as soon as S is
// done, V once the previous tile's O store has read the stage (O is staged
// in the V stage and written by TMA store).  Every mbarrier wait is bounded; a group
// leaves its loop together (the barrier that closes each step ANDs the
// threads' wait results) and drains what it issued before TMEM is freed.
#pragma once

#include "attn_temporal.cuh"

namespace va3d {
namespace tpc {

using tp::TemporalArgs;

constexpr int kThreads = 256;
constexpr int kHalfBytes = 16384;      // 128 rows x 128 B (one 64-dim half)
constexpr int kTensorBytes = 32768;    // 128 rows x 256 B
constexpr int OFF_QK = 0;              // group g: Q at 65536 g, K at 65536 g + 32768
constexpr int OFF_V = 131072;          // group g: V at OFF_V + 32768 g
constexpr int OFF_TAB = 196608;        // t angles, frame-major
constexpr int kMiscBytes = 256;        // barriers, reduction slots, TMEM slot, abort flag
constexpr int kTmemCols = 512;         // group g: S/O at 256 g, P at 256 g + 128

// per group: Q/K landed, V landed, S done, O done, the bf16 k-steps of S done
// (issued before the t range is turned), drain on the way out
enum Bar { B_QK0 = 0, B_V0 = 2, B_S0 = 4, B_O0 = 6, B_E0 = 8, B_DRAIN0 = 10, NUM_BARS = 12 };

// Pairs per frame in the shared angle table: the turned region's pairs
// (ceil16(d_t) dims), identity past the t pairs.  A frame's row is padded by
// one 16-byte slot, so its stride is an odd number of 16-byte units and the
// 16-byte reads of eight consecutive frames fall in eight distinct bank
// groups.
__host__ __device__ inline int tab_pairs(int pe_t) { return ((2 * pe_t + 15) / 16) * 8; }

__host__ __device__ inline int tab_stride(int pe_t) { return tab_pairs(pe_t) + 2; }

__host__ __device__ inline int tab_bytes(int T, int pe_t) { return T * tab_stride(pe_t) * 8; }

// Keys that come rotated: per warp, the h and w angles of its (up to four)
// positions, 64 pairs each.
constexpr int kHwBytes = 8 * 4 * 64 * 8;

__host__ inline int smem_bytes(int T, int pe_t, bool raw_k) {
    return 1024 + OFF_TAB + tab_bytes(T, pe_t) + kMiscBytes + (raw_k ? 0 : kHwBytes);
}

__host__ __device__ constexpr int rows_per_position(int T) { return T <= 8 ? 8 : (T <= 16 ? 16 : 32); }

template <int R>
struct Geo {
    static_assert(R == 8 || R == 16 || R == 32, "R divides 32");
    static constexpr int P = 128 / R;       // positions per tile
    static constexpr int KMAX = 32 / R - 1; // positions after a warp's first one
};

__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) { return smem_desc_sw128(saddr, 16, 1024); }

__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr) {
    return smem_desc_sw128(saddr, kHalfBytes, 1024);
}

// Byte offset of 16-byte chunk c (0..15) of tile row r in a staged tensor
// (two 64-dim halves, 128-byte swizzle as the TMA writes it).
__device__ __forceinline__ uint32_t chunk_off(int r, int c) {
    return static_cast<uint32_t>((c >> 3) * kHalfBytes + r * 128 + ((((c & 7) ^ (r & 7))) << 4));
}

__device__ __forceinline__ float absmax8(uint4 x, float m) {
    const float2 a = unpack_bf16x2(x.x), b = unpack_bf16x2(x.y), c = unpack_bf16x2(x.z),
                 d = unpack_bf16x2(x.w);
    m = fmax3(m, fabsf(a.x), fabsf(a.y));
    m = fmax3(m, fabsf(b.x), fabsf(b.y));
    m = fmax3(m, fabsf(c.x), fabsf(c.y));
    return fmax3(m, fabsf(d.x), fabsf(d.y));
}

// Maximum / sum of n values as a pairwise tree (short dependency chains).
template <int n>
__device__ __forceinline__ float tree_max(float (&x)[n]) {
#pragma unroll
    for (int w = n; w > 1; w = (w + 1) / 2) {
#pragma unroll
        for (int i = 0; i < w / 2; ++i) x[i] = fmaxf(x[i], x[i + (w + 1) / 2]);
    }
    return x[0];
}

template <int n>
__device__ __forceinline__ float tree_sum(float (&x)[n]) {
#pragma unroll
    for (int w = n; w > 1; w = (w + 1) / 2) {
#pragma unroll
        for (int i = 0; i < w / 2; ++i) x[i] += x[i + (w + 1) / 2];
    }
    return x[0];
}

// Softmax of one row over its position's key columns.  sv: the warp's 32
// columns of S (position k of the warp at columns [k R, k R + R)); the row's
// position is `kofs`; only its first C columns are read (C >= T', the rest
// are padding).  Writes the warp's 16 P words (bf16 pairs, zero outside the
// row's block) and returns 1 / (row sum).
template <int R, int C>
__device__ __forceinline__ float softmax_block(const uint32_t (&sv)[32], int T, int kofs, float sl,
                                               uint32_t (&w)[16]) {
    constexpr int KMAX = 32 / R - 1;
    float s[C], t[C];
#pragma unroll
    for (int i = 0; i < C; ++i) {
        uint32_t v = sv[i];
#pragma unroll
        for (int k = 1; k <= KMAX; ++k)
            if (kofs == k) v = sv[i + k * R];
        s[i] = i < T ? __uint_as_float(v) : -INFINITY;
        t[i] = s[i];
    }
    const float nm = -tree_max(t) * sl;
#pragma unroll
    for (int i = 0; i < C; ++i) {
        s[i] = ex2(fmaf(s[i], sl, nm));
        t[i] = s[i];
    }
    const float inv_l = 1.0f / tree_sum(t);
    uint32_t pk[C / 2];
#pragma unroll
    for (int j = 0; j < C / 2; ++j) pk[j] = pack_bf16x2(s[2 * j], s[2 * j + 1]);
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = 0u;
#pragma unroll
    for (int k = 0; k <= KMAX; ++k)
        if (kofs == k) {
#pragma unroll
            for (int j = 0; j < C / 2; ++j) w[k * (R / 2) + j] = pk[j];
        }
    return inv_l;
}

template <int R, bool kRawK>
__global__ void __launch_bounds__(kThreads, 1)
temporal_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const __grid_constant__ TemporalArgs a) {
    using G = Geo<R>;
    constexpr int P = G::P, KMAX = G::KMAX;
    constexpr uint32_t kBoxBytes = 64u * R * P * 2u;
    constexpr uint32_t kIdBf16 = idesc_bf16_f32(128, 128, 0);
    constexpr uint32_t kIdF16 = idesc_f16_f32(128, 128);
    constexpr uint32_t kIdPV = idesc_bf16_f32(128, 128, 1);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const uint32_t sbase = smem_u32(smem);
    const int T = a.T;
    const int TP = tab_pairs(a.rp.pe_t);
    const int TS = tab_stride(a.rp.pe_t);
    const int nc = TP / 4;                     // 16-byte chunks of the fp16 region (even)
    const int off_misc = OFF_TAB + tab_bytes(T, a.rp.pe_t);
    float2 *tab = reinterpret_cast<float2 *>(smem + OFF_TAB);
    uint8_t *misc = smem + off_misc;
    float2 *hw_ang = reinterpret_cast<float2 *>(misc + kMiscBytes);   // [warp][position][pair]
    auto bar = [&](int i) -> uint32_t { return sbase + off_misc + 8 * i; };
    float *red = reinterpret_cast<float *>(misc + 128);   // [group][warp][2]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 200);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = warp >> 2, wl = warp & 3;
    const int r = wl * 32 + lane;             // tile row = TMEM lane
    const bool leader = (threadIdx.x & 127) == 0;
    const int p_loc = r / R;                  // local position of this row
    const int f = r - p_loc * R;              // frame of this row
    const int kofs = p_loc - (wl * 32) / R;   // position within the warp's: 0..KMAX

    const int tiles_per_bh = (a.HW + P - 1) / P;
    const int n_tiles = a.BH * tiles_per_bh;   // the launcher keeps this below 2^31

    if (threadIdx.x == 0) {
        for (int i = 0; i < NUM_BARS; ++i) mbar_init(bar(i), 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    // the t angles of each frame (identity past the t pairs)
    for (int i = threadIdx.x; i < T * TS; i += kThreads) {
        const int ff = i / TS, j = i - ff * TS;
        tab[i] = j < a.rp.pe_t ? a.rope_tab[j * T + ff] : make_float2(1.f, 0.f);
    }
    if (warp == 0) tmem_alloc(sbase + off_misc + 192, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(misc + 192);
    const uint32_t lane_addr = static_cast<uint32_t>(wl * 32) << 16;
    const uint32_t colS = 256u * g;           // S, then O
    const uint32_t colP = 256u * g + 128u;    // P as bf16 pairs
    {
        uint32_t z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_st32(tmem + lane_addr + colP + 32 * c, z);
        tmem_wait_st();
    }

    const uint32_t Qs = sbase + OFF_QK + 65536u * g, Ks = Qs + kTensorBytes;
    const uint32_t Vs = sbase + OFF_V + static_cast<uint32_t>(kTensorBytes) * g;
    uint8_t *sq = smem + OFF_QK + 65536 * g;
    uint8_t *sk = sq + kTensorBytes;
    uint8_t *sv = smem + OFF_V + kTensorBytes * g;   // V, then O staged for the store
    const int bid = 1 + g;                    // this group's named barrier

    // group g takes the CTA's tiles 2n + g
    auto tile_of = [&](int n) -> int { return static_cast<int>(blockIdx.x) + (2 * n + g) * static_cast<int>(gridDim.x); };
    auto load_qk = [&](int bh, int pos0) {
        mbar_arrive_expect_tx(bar(B_QK0 + g), 4u * kBoxBytes);
        tma_load_4d(Qs, &tmQ, bar(B_QK0 + g), 0, 0, pos0, bh);
        tma_load_4d(Qs + kHalfBytes, &tmQ, bar(B_QK0 + g), 64, 0, pos0, bh);
        tma_load_4d(Ks, &tmK, bar(B_QK0 + g), 0, 0, pos0, bh);
        tma_load_4d(Ks + kHalfBytes, &tmK, bar(B_QK0 + g), 64, 0, pos0, bh);
    };
    auto load_v = [&](int bh, int pos0) {
        mbar_arrive_expect_tx(bar(B_V0 + g), 2u * kBoxBytes);
        tma_load_4d(Vs, &tmV, bar(B_V0 + g), 0, 0, pos0, bh);
        tma_load_4d(Vs + kHalfBytes, &tmV, bar(B_V0 + g), 64, 0, pos0, bh);
    };

    // leader: loads issued and not yet seen complete (drained on the way out)
    bool qk_out = false, v_out = false;
    uint32_t qk_ph = 0, v_ph = 0;
    int t = tile_of(0);
    int bh = t / tiles_per_bh;
    int pos0 = (t - bh * tiles_per_bh) * P;
    if (leader && t < n_tiles) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmO);
        load_qk(bh, pos0);
        load_v(bh, pos0);
        qk_out = v_out = true;
    }

    bool good = true;   // every wait of this warp so far succeeded (warp-uniform)
    // The second group starts once the first group's first S is done, so the
    // two run half a step apart (one's arithmetic over the other's products)
    // rather than in step.
    if (g == 1)
        good = __all_sync(0xffffffffu, mbar_wait(bar(B_S0), 0, abort_flag, VA3D_DEVERR_TIMEOUT_SOFTMAX));
    for (int n = 0; t < n_tiles; ++n) {
        const uint32_t ph = static_cast<uint32_t>(n & 1);
        const int t2 = tile_of(n + 1);   // this group's next tile
        const int bh2 = t2 / tiles_per_bh;
        const int pos02 = (t2 - bh2 * tiles_per_bh) * P;
        const int pos = pos0 + p_loc;
        const bool valid = f < T && p_loc < P && pos < a.HW;
        const size_t rowofs =
            valid ? (static_cast<size_t>(bh) * a.N + static_cast<size_t>(f) * a.HW + pos) * 128 : 0;  // full path

        // ---- Q and K of this tile have landed
        if (good) {
            const bool mine = mbar_wait(bar(B_QK0 + g), ph, abort_flag, VA3D_DEVERR_TIMEOUT_SOFTMAX);
            if (leader && mine) qk_out = false;
            good = __all_sync(0xffffffffu, mine);
        }
        if (leader && good) {
            tc_fence_after();
            if constexpr (kRawK) {
                // the k-steps past the t range read untouched inputs: start
                // them now, under the turning below (the previous tile's O
                // was read out before the barrier that ended it)
#pragma unroll 1
                for (int kk = nc / 2; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + colS, desc_kmajor(Qs + off), desc_kmajor(Ks + off), kIdBf16,
                           kk > nc / 2 ? 1u : 0u);
                }
                mma_commit(bar(B_E0 + g));
            }
            // this tile's V (the previous tile's O store has read the stage)
            if (n > 0) {
                bulk_wait_group_read0();
                load_v(bh, pos0);
                v_out = true;
                v_ph = ph;
            }
        }
        // ---- raw keys: turn the t range of this row of Q and K in place (fp16).
        // Keys that come rotated: turn all of this row of Q and convert K,
        // both unscaled fp16.  mx tracks the largest value written.
        float mx = 0.f;
        if (!kRawK && good) {
            // the h and w angles of this row's position, computed once by its
            // R rows (hardware sine and cosine: absolute error ~1e-5 at the
            // largest angles of the pages' grids, far below fp16's rounding of
            // the turned values)
            const int hh = pos / a.rp.W, ww = pos - hh * a.rp.W;
            const float fh = static_cast<float>(hh), fw = static_cast<float>(ww);
            float2 *ha = hw_ang + (warp * 4 + kofs) * 64;
            for (int p = a.rp.pe_t + f; p < 64; p += R) {
                float2 cs;
                __sincosf((p < a.rp.pe_h ? fh : fw) * a.rp.inv_freq[p], &cs.y, &cs.x);
                ha[p] = cs;
            }
            __syncwarp();
        }
        if (!kRawK && good && valid) {
            const float2 *ha = hw_ang + (warp * 4 + kofs) * 64;
            const float2 *tt = tab + f * TS;
            float m2[2] = {0.f, 0.f};
            for (int c = 0; c < 16; c += 2) {
                // two chunks per pass: all loads first
                uint4 xq[2], xk[2];
                float2 cq[2][4];
                uint32_t off[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    off[u] = chunk_off(r, c + u);
                    xq[u] = *reinterpret_cast<const uint4 *>(sq + off[u]);
                    xk[u] = *reinterpret_cast<const uint4 *>(sk + off[u]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int p = 4 * (c + u) + e;
                        cq[u][e] = p < a.rp.pe_t ? tt[p] : ha[p];
                    }
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    *reinterpret_cast<uint4 *>(sq + off[u]) = make_uint4(
                        tp::rot_f16_max(xq[u].x, cq[u][0], m2[u]), tp::rot_f16_max(xq[u].y, cq[u][1], m2[u]),
                        tp::rot_f16_max(xq[u].z, cq[u][2], m2[u]), tp::rot_f16_max(xq[u].w, cq[u][3], m2[u]));
                    *reinterpret_cast<uint4 *>(sk + off[u]) = make_uint4(
                        tp::cvt_f16_max(xk[u].x, m2[u]), tp::cvt_f16_max(xk[u].y, m2[u]),
                        tp::cvt_f16_max(xk[u].z, m2[u]), tp::cvt_f16_max(xk[u].w, m2[u]));
                }
            }
            mx = fmaxf(m2[0], m2[1]);
        }
        if (kRawK && good && valid) {
            const float2 *ang = tab + f * TS;
            for (int c = 0; c < nc; c += 2) {
                // two chunks per pass: all loads first
                uint4 vq[2], vk[2];
                float4 an[4];
                uint32_t off[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    off[u] = chunk_off(r, c + u);
                    vq[u] = *reinterpret_cast<const uint4 *>(sq + off[u]);
                    vk[u] = *reinterpret_cast<const uint4 *>(sk + off[u]);
                    an[2 * u] = *reinterpret_cast<const float4 *>(ang + 4 * (c + u));
                    an[2 * u + 1] = *reinterpret_cast<const float4 *>(ang + 4 * (c + u) + 2);
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const float2 c0 = make_float2(an[2 * u].x, an[2 * u].y);
                    const float2 c1 = make_float2(an[2 * u].z, an[2 * u].w);
                    const float2 c2 = make_float2(an[2 * u + 1].x, an[2 * u + 1].y);
                    const float2 c3 = make_float2(an[2 * u + 1].z, an[2 * u + 1].w);
                    *reinterpret_cast<uint4 *>(sq + off[u]) =
                        make_uint4(tp::rot_f16_max(vq[u].x, c0, mx), tp::rot_f16_max(vq[u].y, c1, mx),
                                   tp::rot_f16_max(vq[u].z, c2, mx), tp::rot_f16_max(vq[u].w, c3, mx));
                    *reinterpret_cast<uint4 *>(sk + off[u]) =
                        make_uint4(tp::rot_f16_max(vk[u].x, c0, mx), tp::rot_f16_max(vk[u].y, c1, mx),
                                   tp::rot_f16_max(vk[u].z, c2, mx), tp::rot_f16_max(vk[u].w, c3, mx));
                }
            }
        }
        {
            const uint32_t wm = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
            if (lane == 0) red[(g * 4 + wl) * 2] = __uint_as_float(wm);
        }
        fence_proxy_async_smem();
        if (!named_and(bid, 128, good)) break;
        int f16_steps = kRawK ? nc / 2 : 8;   // k-steps of QK^T over fp16 operands
        int eq = 0, ek = 0;
        const bool full = !tp::fp16_range_ok(
            fmaxf(fmaxf(red[g * 8], red[g * 8 + 2]), fmaxf(red[g * 8 + 4], red[g * 8 + 6])));
        if (full) {
            // the values written left fp16's comfortable range: all dims in
            // fp16 under per-tile powers of two, from the rows in global memory
            // (the stage holds turned values), once the early bf16 products
            // have read the stage
            if constexpr (kRawK)
                good = __all_sync(0xffffffffu, mbar_wait(bar(B_E0 + g), ph, abort_flag,
                                                         VA3D_DEVERR_TIMEOUT_SOFTMAX)) && good;
            const __nv_bfloat16 *gq = a.q + rowofs, *gk = a.k + rowofs;
            auto row_q = [&](int c) -> uint4 { return tp::ldg_stream(gq + 8 * c); };
            auto row_k = [&](int c) -> uint4 { return tp::ldg_stream(gk + 8 * c); };
            float mq = 0.f, mk = 0.f;
            if (valid) {
#pragma unroll 4
                for (int c = 0; c < 16; ++c) {
                    mq = absmax8(row_q(c), mq);
                    mk = absmax8(row_k(c), mk);
                }
            }
            const uint32_t wq = __reduce_max_sync(0xffffffffu, __float_as_uint(mq));
            const uint32_t wk = __reduce_max_sync(0xffffffffu, __float_as_uint(mk));
            // the slots were read by every thread before the barrier above
            // could be passed a second time: rewrite them after a barrier
            named_sync(bid, 128);
            if (lane == 0) {
                red[(g * 4 + wl) * 2] = __uint_as_float(wq);
                red[(g * 4 + wl) * 2 + 1] = __uint_as_float(wk);
            }
            named_sync(bid, 128);
            float tq = 0.f, tk = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                tq = fmaxf(tq, red[(g * 4 + w) * 2]);
                tk = fmaxf(tk, red[(g * 4 + w) * 2 + 1]);
            }
            eq = tq > 0.f ? tp::fp16_rescale_exponent(tq) : 0;
            ek = tk > 0.f ? tp::fp16_rescale_exponent(tk) : 0;
            const float sq_scale = tp::pow2f(eq), sk_scale = tp::pow2f(ek);
            if (valid) {
                const int hh = pos / a.rp.W, ww = pos - hh * a.rp.W;
#pragma unroll 2
                for (int c = 0; c < 16; ++c) {
                    const uint4 xq = row_q(c);
                    const uint4 xk = row_k(c);
                    float2 cq[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int p = 4 * c + e;
                        float2 an;
                        if (p < a.rp.pe_t)
                            an = tab[f * TS + p];
                        else if (kRawK)
                            an = make_float2(1.f, 0.f);
                        else   // same address across a position's rows: a broadcast
                            an = __ldg(&a.rope_tab[table_index(a.rp, p, 0, hh, ww)]);
                        cq[e] = make_float2(an.x * sq_scale, an.y * sq_scale);
                    }
                    const uint32_t off = chunk_off(r, c);
                    *reinterpret_cast<uint4 *>(sq + off) =
                        make_uint4(tp::rot_f16(xq.x, cq[0]), tp::rot_f16(xq.y, cq[1]),
                                   tp::rot_f16(xq.z, cq[2]), tp::rot_f16(xq.w, cq[3]));
                    if constexpr (kRawK) {
                        // raw keys: t pairs turned, the others converted
                        float2 ck[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int p = 4 * c + e;
                            const float2 bk = p < a.rp.pe_t ? tab[f * TS + p] : make_float2(1.f, 0.f);
                            ck[e] = make_float2(bk.x * sk_scale, bk.y * sk_scale);
                        }
                        *reinterpret_cast<uint4 *>(sk + off) =
                            make_uint4(tp::rot_f16(xk.x, ck[0]), tp::rot_f16(xk.y, ck[1]),
                                       tp::rot_f16(xk.z, ck[2]), tp::rot_f16(xk.w, ck[3]));
                    } else {
                        *reinterpret_cast<uint4 *>(sk + off) =
                            make_uint4(tp::cvt_f16(xk.x, sk_scale), tp::cvt_f16(xk.y, sk_scale),
                                       tp::cvt_f16(xk.z, sk_scale), tp::cvt_f16(xk.w, sk_scale));
                    }
                }
            }
            fence_proxy_async_smem();
            named_sync(bid, 128);
            f16_steps = 8;
        }
        const float sl = a.scale_log2 * tp::pow2f(-(eq + ek));

        // ---- S = Q K^T: the fp16 k-steps (all eight on the full path, which
        // starts the sum again)
        if (leader) {
            tc_fence_after();
            const bool added = kRawK && !full && nc / 2 < 8;   // early bf16 steps in S
#pragma unroll 1
            for (int kk = 0; kk < f16_steps; ++kk) {
                const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                mma_ss(tmem + colS, desc_kmajor(Qs + off), desc_kmajor(Ks + off), kIdF16,
                       (added || kk > 0) ? 1u : 0u);
            }
            mma_commit(bar(B_S0 + g));
        }
        good = __all_sync(0xffffffffu, mbar_wait(bar(B_S0 + g), ph, abort_flag, VA3D_DEVERR_TIMEOUT_SOFTMAX));
        tc_fence_after();
        // the Q/K stage is free: the leader loads this group's next tile into it
        if (leader && good && t2 < n_tiles) {
            load_qk(bh2, pos02);
            qk_out = true;
            qk_ph = ph ^ 1u;
        }

        // ---- softmax over the row's keys; P into the warp's 16 columns
        float inv_l = 0.f;
        if (good) {
            uint32_t sv[32];
            tmem_ld32(tmem + lane_addr + colS + 32u * wl, sv);
            tmem_wait_ld();
            reg_fence32(sv);
            uint32_t w[16];
            if constexpr (R == 32) {
                // frames 24..31 are padding unless T' > 24
                if (T <= 24)
                    inv_l = softmax_block<R, 24>(sv, T, kofs, sl, w);
                else
                    inv_l = softmax_block<R, 32>(sv, T, kofs, sl, w);
            } else {
                inv_l = softmax_block<R, R>(sv, T, kofs, sl, w);
            }
            tmem_st16(tmem + lane_addr + colP + 16u * wl, w);
            tmem_wait_st();
        }
        tc_fence_before();
        if (!named_and(bid, 128, good)) break;

        // ---- O = P V into the S columns
        if (leader) {
            tc_fence_after();
            if (mbar_wait(bar(B_V0 + g), ph, abort_flag, VA3D_DEVERR_TIMEOUT_MMA)) {
                v_out = false;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + colS, tmem + colP + 8 * kk, desc_mnmajor(Vs + kk * 2048), kIdPV,
                           kk > 0 ? 1u : 0u);
                mma_commit(bar(B_O0 + g));
            }
            // on a timeout the abort flag ends the others' wait below
        }
        good = __all_sync(0xffffffffu, mbar_wait(bar(B_O0 + g), ph, abort_flag, VA3D_DEVERR_TIMEOUT_SOFTMAX));
        tc_fence_after();

        // ---- O rows: normalise, round to bf16, stage them in the (now free) V
        // stage in the layout the loads use; the leader stores the tile with
        // two TMA boxes (frames past T' and positions past H'W' are clipped)
        if (good) {
            const float2 il2 = make_float2(inv_l, inv_l);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t o0[32], o1[32];
                tmem_ld32(tmem + lane_addr + colS + 64 * hh, o0);
                tmem_ld32(tmem + lane_addr + colS + 64 * hh + 32, o1);
                tmem_wait_ld();
                reg_fence32(o0);
                reg_fence32(o1);
                auto pk2 = [&](const uint32_t *x) {
                    const float2 y = tp::mul2(make_float2(__uint_as_float(x[0]), __uint_as_float(x[1])), il2);
                    return pack_bf16x2(y.x, y.y);
                };
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    *reinterpret_cast<uint4 *>(sv + chunk_off(r, 8 * hh + q4)) =
                        make_uint4(pk2(o0 + 8 * q4), pk2(o0 + 8 * q4 + 2), pk2(o0 + 8 * q4 + 4), pk2(o0 + 8 * q4 + 6));
                    *reinterpret_cast<uint4 *>(sv + chunk_off(r, 8 * hh + 4 + q4)) =
                        make_uint4(pk2(o1 + 8 * q4), pk2(o1 + 8 * q4 + 2), pk2(o1 + 8 * q4 + 4), pk2(o1 + 8 * q4 + 6));
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        if (!named_and(bid, 128, good)) break;
        if (leader) {
            tma_store_4d(&tmO, Vs, 0, 0, pos0, bh);
            tma_store_4d(&tmO, Vs + kHalfBytes, 64, 0, pos0, bh);
            bulk_commit_group();
            // the stage is loaded again (next tile) once the store has read it
        }
        t = t2;
        bh = bh2;
        pos0 = pos02;
    }

    // products and loads this group issued finish before TMEM and shared
    // memory are given up
    if (leader) {
        bulk_wait_group_read0();   // the last O store has read its stage
        mma_commit(bar(B_DRAIN0 + g));
        mbar_wait_drain(bar(B_DRAIN0 + g), 0);
        if (qk_out) mbar_wait_drain(bar(B_QK0 + g), qk_ph);
        if (v_out) mbar_wait_drain(bar(B_V0 + g), v_ph);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tpc
}  // namespace va3d

// Temporal pass of factorised attention (handbook "How attention sees time":
// at each spatial position, attention along time over H'W' sequences of T'
// tokens).  Token (t, h, w) of a sequence sits at row t*H'W' + h*W' + w, so a
// position's T' rows are H'W' rows apart.
//
// The pass is HBM-bound (each position reads T' rows of Q, K, V and writes T'
// rows of O; its 4*T'^2*d FLOPs are small), so the design goal is streaming:
//  - persistent warps (up to 14 per block for T' <= 32, 12 for T' <= 64; as
//    many as shared memory holds), one
//    (batch*head, position) task at a time, rows fetched with 16-byte
//    cp.async (each row is 256 contiguous bytes); the other resident warps
//    compute while one waits for its rows;
//  - only the T' real rows are staged; m16n8k16 fragments that reach past
//    row T'-1 read row T'-1 again (their scores are masked or their outputs
//    dropped), so nothing is zero-filled;
//  - raw keys (the usual call): within one position every row has the same
//    (h, w), so the h and w rotations of Q and K cancel in q.k and only the
//    t range needs turning.  The first ceil16(d_t) dims of Q and K are turned
//    (t pairs) and stored as fp16 in place; the remaining dims stay the raw
//    bf16 inputs, whose products are exact.  QK^T then runs fp16 MMAs on the
//    first k-steps and bf16 MMAs on the rest, into one fp32 accumulator.  The
//    rotated operands are never rounded to bf16: the temporal softmax has
//    only T' terms, its outputs are O(1), and such rounding would dominate the
//    error.  If the turned values leave fp16's comfortable range the task is
//    redone with all dims in fp16 under a power-of-two scale;
//  - keys that come rotated: Q is turned in full, both are stored as fp16
//    scaled by powers of two, and QK^T runs fp16 MMAs throughout;
//  - S = Q K^T (fp16) and O = P V (bf16) on the m16n8k16 tensor-core path with
//    fp32 accumulation; O staged through shared memory for 16-byte row stores.
#pragma once

#include <cuda_fp16.h>

#include "ptx.cuh"
#include "rope.cuh"

namespace va3d {
namespace tp {

struct TemporalArgs {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;
    __nv_bfloat16 *o;
    int N;                     // tokens per sequence (T*HW)
    int T;                     // frames T'
    int HW;                    // positions per frame H'W'
    int BH;                    // batch * heads
    float scale_log2;          // softmax scale * log2(e)
    int rope_k;                // 1: k holds raw keys, rotate them here
    const float2 *rope_tab;
    RopeParams rp;
};

// Byte offset of 16-byte chunk c (0..15) of row r in a 256-byte-row tile:
// the low three chunk bits are XORed with the row so that the eight rows an
// ldmatrix reads fall in distinct bank groups.
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return static_cast<uint32_t>(r * 256 + (((c & 8) | ((c ^ r) & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float pow2f(int s) {
    return __uint_as_float(static_cast<uint32_t>(127 + s) << 23);
}

template <int MAXT>
struct Cfg {
    // T' <= 32: up to 14 warps (128 registers each, no spills; at T' = 21
    // their Q, K, V take 226 KB).  T' <= 64: up to 12 warps (168 registers);
    // at T' = 64 shared memory holds 4.
    static constexpr int kMaxWarps = MAXT <= 32 ? 14 : 12;
    static constexpr int kSmemBudget = (MAXT <= 32 ? 226 : 208) * 1024;
};

// Shared memory per warp: (Q, K, V) with T rows of 256 bytes.
__host__ __device__ inline int temporal_warp_bytes(int T) { return 3 * T * 256; }

// Shared memory for the block's copy of the angle table's t section
// (T * d_t/2 (cos, sin) pairs), rounded up to 16 bytes.
__host__ __device__ inline int temporal_table_bytes(int T, int half_t) {
    return (T * half_t * 8 + 15) / 16 * 16;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// One rotated pair (x0 c - x1 s, x0 s + x1 c) times a power-of-two scale,
// where cs holds (c * scale, s * scale); returned as packed fp16.  m tracks
// the largest magnitude of the unscaled rotated values (cs / scale).
__device__ __forceinline__ uint32_t rot_f16(uint32_t packed_bf16, float2 cs) {
    const float2 x = unpack_bf16x2(packed_bf16);
    const float2 y = fma2(x, make_float2(cs.x, cs.x), mul2(make_float2(-x.y, x.x), make_float2(cs.y, cs.y)));
    return pack_f16x2(y.x, y.y);
}

__device__ __forceinline__ uint32_t rot_f16_max(uint32_t packed_bf16, float2 cs, float &m) {
    const float2 x = unpack_bf16x2(packed_bf16);
    const float2 y = fma2(x, make_float2(cs.x, cs.x), mul2(make_float2(-x.y, x.x), make_float2(cs.y, cs.y)));
    m = fmax3(m, fabsf(y.x), fabsf(y.y));
    return pack_f16x2(y.x, y.y);
}

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// fp16 is used as is when the largest rotated magnitude lies in
// [2^-6, 2^15); outside that range the operand is redone with a power of two
// that brings its largest magnitude into [2^13, 2^14).
__device__ __forceinline__ bool fp16_range_ok(float m) {
    return m == 0.0f || (m >= 0.015625f && m < 32768.0f);
}

__device__ __forceinline__ int fp16_rescale_exponent(float m) {
    const int e = static_cast<int>((__float_as_uint(m) >> 23) & 0xFF) - 127;   // m in [2^e, 2^(e+1))
    return max(-60, min(60, 13 - e));
}

// A bf16 pair as packed fp16 times a power of two (no rotation); m tracks the
// largest magnitude of the unscaled values.
__device__ __forceinline__ uint32_t cvt_f16_max(uint32_t packed_bf16, float &m) {
    const float2 x = unpack_bf16x2(packed_bf16);
    m = fmax3(m, fabsf(x.x), fabsf(x.y));
    return pack_f16x2(x.x, x.y);
}

__device__ __forceinline__ uint32_t cvt_f16(uint32_t packed_bf16, float sc) {
    const float2 x = unpack_bf16x2(packed_bf16);
    return pack_f16x2(x.x * sc, x.y * sc);
}

// RoPE (when kRotate; keys that come rotated are only converted) + fp16 in
// place for the T rows of one staged operand (raw bf16 rows in shared
// memory).  Scale 1 unless the largest magnitude is out of fp16's
// comfortable range; then the rows are read again from global memory and
// redone with a power-of-two scale, whose exponent is returned.
template <bool kRotate>
__device__ __forceinline__ int rotate_to_f16(uint8_t *tile, const __nv_bfloat16 *src, size_t base,
                                             size_t tstride, int T, int rlane, int cch,
                                             const float2 (&cs_fixed)[4], const bool (&is_t)[4],
                                             const float2 *t_tab) {
    // t pairs: the block's shared copy of the t section (entry j*T + t);
    // h and w pairs: fixed for the task
    auto angle = [&](int r, int e) -> float2 {
        return is_t[e] ? t_tab[(cch * 4 + e) * T + r] : cs_fixed[e];
    };
    float mx = 0.f;
    for (int r = rlane; r < T; r += 2) {
        uint4 *p = reinterpret_cast<uint4 *>(tile + swz(r, cch));
        const uint4 x = *p;
        if constexpr (kRotate)
            *p = make_uint4(rot_f16_max(x.x, angle(r, 0), mx), rot_f16_max(x.y, angle(r, 1), mx),
                            rot_f16_max(x.z, angle(r, 2), mx), rot_f16_max(x.w, angle(r, 3), mx));
        else
            *p = make_uint4(cvt_f16_max(x.x, mx), cvt_f16_max(x.y, mx), cvt_f16_max(x.z, mx),
                            cvt_f16_max(x.w, mx));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (fp16_range_ok(mx)) return 0;
    const int ex = fp16_rescale_exponent(mx);
    const float sc = pow2f(ex);
    for (int r = rlane; r < T; r += 2) {
        const uint4 x = ldg_stream(src + base + r * tstride + cch * 8);
        if constexpr (kRotate) {
            float2 c[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                c[e] = angle(r, e);
                c[e] = make_float2(c[e].x * sc, c[e].y * sc);
            }
            *reinterpret_cast<uint4 *>(tile + swz(r, cch)) =
                make_uint4(rot_f16(x.x, c[0]), rot_f16(x.y, c[1]), rot_f16(x.z, c[2]), rot_f16(x.w, c[3]));
        } else {
            *reinterpret_cast<uint4 *>(tile + swz(r, cch)) =
                make_uint4(cvt_f16(x.x, sc), cvt_f16(x.y, sc), cvt_f16(x.z, sc), cvt_f16(x.w, sc));
        }
    }
    return ex;
}

// Raw keys: the first nc 16-byte chunks of every Q and K row (dims 0 .. 8nc-1,
// nc = ceil16(d_t) / 8) turned by their t angles (pairs past the t range are
// kept) and stored as unscaled fp16 in place.  Lane (rr, cc) = (lane / nc,
// lane % nc) takes chunk cc of rows rr, rr + rpi, ...  Returns the largest
// magnitude written (for the fp16 range check).
__device__ __forceinline__ float turn_t_region(uint8_t *qt, uint8_t *kt, int T, int lane, int nc, int rpi,
                                               int pe_t, const float2 *t_tab) {
    float mx = 0.f;
    if (lane >= rpi * nc) return mx;
    const int rr = lane / nc;
    const int cc = lane - rr * nc;
    for (int r = rr; r < T; r += rpi) {
        uint4 *pq = reinterpret_cast<uint4 *>(qt + swz(r, cc));
        uint4 *pk = reinterpret_cast<uint4 *>(kt + swz(r, cc));
        const uint4 vq = *pq, vk = *pk;
        float2 c[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int p = cc * 4 + e;
            c[e] = p < pe_t ? t_tab[p * T + r] : make_float2(1.f, 0.f);
        }
        *pq = make_uint4(rot_f16_max(vq.x, c[0], mx), rot_f16_max(vq.y, c[1], mx),
                         rot_f16_max(vq.z, c[2], mx), rot_f16_max(vq.w, c[3], mx));
        *pk = make_uint4(rot_f16_max(vk.x, c[0], mx), rot_f16_max(vk.y, c[1], mx),
                         rot_f16_max(vk.z, c[2], mx), rot_f16_max(vk.w, c[3], mx));
    }
    return mx;
}

// kRawK: k holds raw keys (a.rope_k == 1); otherwise the keys come rotated.
template <int MAXT, bool kRawK>
__global__ void __launch_bounds__(Cfg<MAXT>::kMaxWarps * 32)
temporal_kernel(const __grid_constant__ TemporalArgs a) {
    constexpr int NP = MAXT / 16;   // pairs of n8 key tiles and k16 key steps
    constexpr int MG = 2;           // query m-tiles computed together
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int T = a.T;
    const int tensor_bytes = T * 256;
    const long long total = static_cast<long long>(a.BH) * a.HW;
    const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
    long long task = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + warp;

    // The t angles vary per row of every task: the block keeps a copy of the
    // table's t section in shared memory (read-only after this barrier, the
    // only block-wide barrier).
    float2 *t_tab = reinterpret_cast<float2 *>(smem);
    const int n_t = T * a.rp.half_t;
    for (int i = threadIdx.x; i < n_t; i += blockDim.x) t_tab[i] = a.rope_tab[i];
    __syncthreads();
    if (task >= total) return;   // the whole warp leaves together

    uint8_t *sq = smem + temporal_table_bytes(T, a.rp.half_t) + warp * temporal_warp_bytes(T);
    // sq: Q (raw, fp16 rotated, then bf16 O)
    uint8_t *sk = sq + tensor_bytes;                     // K (raw, then fp16 rotated)
    uint8_t *sv = sk + tensor_bytes;                     // V (bf16)
    const uint32_t aq = smem_u32(sq), ak = smem_u32(sk), av = smem_u32(sv);
    const size_t tstride = static_cast<size_t>(a.HW) * 128;   // elements between frames

    const int g = lane >> 2;      // mma fragment row
    const int tq = lane & 3;      // mma fragment column pair
    // In the copy and rotate passes lane handles 16-byte chunk cch (pairs
    // 4cch..4cch+3) of rows rlane, rlane + 2, ...
    const int cch = lane & 15;
    const int rlane = lane >> 4;
    const int tl = T - 1;
    const int n_mt = (T + 15) >> 4;
    // raw keys: the fp16 region is the first nc chunks (ceil16(d_t) dims),
    // i.e. the first kk16 k-steps of QK^T; rpi rows per pass of the warp
    const int nc = ((2 * a.rp.pe_t + 15) / 16) * 2;
    const int kk16 = nc / 2;
    const int rpi = nc > 0 ? 32 / nc : 32;

    for (; task < total; task += stride) {
        const long long bh = task / a.HW;
        const int pos = static_cast<int>(task - bh * a.HW);
        const size_t base = (static_cast<size_t>(bh) * a.N + static_cast<size_t>(pos)) * 128;

        for (int r = rlane; r < T; r += 2) {
            const size_t gofs = base + r * tstride + cch * 8;
            const uint32_t off = swz(r, cch);
            cp_async16(aq + off, a.q + gofs);
            cp_async16(ak + off, a.k + gofs);
            cp_async16(av + off, a.v + gofs);
        }
        cp_async_commit();

        // angles: h and w pairs are fixed for the task, t pairs vary per row
        const int h = pos / a.rp.W;
        const int w = pos - h * a.rp.W;
        float2 cs_fixed[4];
        bool is_t[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int p = cch * 4 + e;
            is_t[e] = p < a.rp.pe_t;
            // h and w angles matter only when Q is turned in full (keys come rotated)
            cs_fixed[e] = is_t[e] || kRawK ? make_float2(1.f, 0.f)
                                            : a.rope_tab[table_index(a.rp, p, 0, h, w)];
        }
        cp_async_wait<0>();
        __syncwarp();
        int eq = 0, ek = 0;
        int f16_steps = 8;   // k-steps of QK^T that read fp16 operands; the rest read bf16
        bool full = !kRawK;
        if constexpr (kRawK) {
            float mx = turn_t_region(sq, sk, T, lane, nc, rpi, a.rp.pe_t, t_tab);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (fp16_range_ok(mx)) {
                f16_steps = kk16;
            } else {
                // out of fp16's comfortable range: all dims to fp16 under a
                // power-of-two scale (t pairs turned, h and w pairs kept).  The
                // first nc chunks were overwritten: fetch them again.
                __syncwarp();
                if (cch < nc) {
                    for (int r = rlane; r < T; r += 2) {
                        const size_t gofs = base + r * tstride + cch * 8;
                        *reinterpret_cast<uint4 *>(sq + swz(r, cch)) = ldg_stream(a.q + gofs);
                        *reinterpret_cast<uint4 *>(sk + swz(r, cch)) = ldg_stream(a.k + gofs);
                    }
                }
                full = true;
            }
            __syncwarp();
        }
        if (full) {
            eq = rotate_to_f16<true>(sq, a.q, base, tstride, T, rlane, cch, cs_fixed, is_t, t_tab);
            ek = rotate_to_f16<kRawK>(sk, a.k, base, tstride, T, rlane, cch, cs_fixed, is_t, t_tab);
        }
        const float scale_log2 = a.scale_log2 * pow2f(-(eq + ek));
        __syncwarp();

        for (int mg = 0; mg < n_mt; mg += MG) {
            // ---- S = Q K^T for query tiles mg, mg+1 (each K fragment loaded once)
            float sacc[MG][2 * NP][4];
#pragma unroll
            for (int m = 0; m < MG; ++m)
#pragma unroll
                for (int nt = 0; nt < 2 * NP; ++nt)
                    sacc[m][nt][0] = sacc[m][nt][1] = sacc[m][nt][2] = sacc[m][nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t af[MG][4];
#pragma unroll
                for (int m = 0; m < MG; ++m)
                    ldsm_x4(aq + swz(min((mg + m) * 16 + (lane & 15), tl), kk * 2 + (lane >> 4)),
                            af[m][0], af[m][1], af[m][2], af[m][3]);
#pragma unroll
                for (int np = 0; np < NP; ++np) {
                    if (np < n_mt) {
                        uint32_t b0, b1, b2, b3;
                        const int krow = min(np * 16 + (lane & 7) + ((lane >> 4) << 3), tl);
                        ldsm_x4(ak + swz(krow, kk * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
                        if (kk < f16_steps) {
#pragma unroll
                            for (int m = 0; m < MG; ++m) {
                                mma_f16(sacc[m][2 * np], af[m][0], af[m][1], af[m][2], af[m][3], b0, b1);
                                mma_f16(sacc[m][2 * np + 1], af[m][0], af[m][1], af[m][2], af[m][3], b2, b3);
                            }
                        } else {
#pragma unroll
                            for (int m = 0; m < MG; ++m) {
                                mma_bf16(sacc[m][2 * np], af[m][0], af[m][1], af[m][2], af[m][3], b0, b1);
                                mma_bf16(sacc[m][2 * np + 1], af[m][0], af[m][1], af[m][2], af[m][3], b2, b3);
                            }
                        }
                    }
                }
            }
            // ---- softmax over the T keys; P as bf16 A fragments
            uint32_t pa[MG][NP][4];
            float il[MG][2];
#pragma unroll
            for (int m = 0; m < MG; ++m) {
                float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 2 * NP; ++nt) {
                    const int c0 = nt * 8 + 2 * tq;
                    if (c0 >= T) { sacc[m][nt][0] = -INFINITY; sacc[m][nt][2] = -INFINITY; }
                    if (c0 + 1 >= T) { sacc[m][nt][1] = -INFINITY; sacc[m][nt][3] = -INFINITY; }
                    m0 = fmax3(m0, sacc[m][nt][0], sacc[m][nt][1]);
                    m1 = fmax3(m1, sacc[m][nt][2], sacc[m][nt][3]);
                }
                m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
                m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
                m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
                m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
                const float nm0 = -m0 * scale_log2, nm1 = -m1 * scale_log2;
                float l0 = 0.f, l1 = 0.f;
#pragma unroll
                for (int nt = 0; nt < 2 * NP; ++nt) {
                    sacc[m][nt][0] = ex2(fmaf(sacc[m][nt][0], scale_log2, nm0));
                    sacc[m][nt][1] = ex2(fmaf(sacc[m][nt][1], scale_log2, nm0));
                    sacc[m][nt][2] = ex2(fmaf(sacc[m][nt][2], scale_log2, nm1));
                    sacc[m][nt][3] = ex2(fmaf(sacc[m][nt][3], scale_log2, nm1));
                    l0 += sacc[m][nt][0] + sacc[m][nt][1];
                    l1 += sacc[m][nt][2] + sacc[m][nt][3];
                }
                l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
                l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
                l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
                l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
                il[m][0] = 1.f / l0;
                il[m][1] = 1.f / l1;
#pragma unroll
                for (int ks = 0; ks < NP; ++ks) {
                    pa[m][ks][0] = pack_bf16x2(sacc[m][2 * ks][0], sacc[m][2 * ks][1]);
                    pa[m][ks][1] = pack_bf16x2(sacc[m][2 * ks][2], sacc[m][2 * ks][3]);
                    pa[m][ks][2] = pack_bf16x2(sacc[m][2 * ks + 1][0], sacc[m][2 * ks + 1][1]);
                    pa[m][ks][3] = pack_bf16x2(sacc[m][2 * ks + 1][2], sacc[m][2 * ks + 1][3]);
                }
            }
            // every lane is done reading these Q rows before O overwrites them
            // (later groups read only higher rows)
            __syncwarp();
            // ---- O = P V, 32 output columns at a time (fewer live accumulators, so
            // more warps fit), staged into the Q rows as bf16
#pragma unroll
            for (int dh = 0; dh < 4; ++dh) {
                float oacc[MG][4][4];
#pragma unroll
                for (int m = 0; m < MG; ++m)
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
                        oacc[m][nt][0] = oacc[m][nt][1] = oacc[m][nt][2] = oacc[m][nt][3] = 0.f;
#pragma unroll
                for (int ks = 0; ks < NP; ++ks) {
                    if (ks < n_mt) {
                        const int vrow = min(ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), tl);
#pragma unroll
                        for (int dp = 0; dp < 2; ++dp) {
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4_t(av + swz(vrow, dh * 4 + dp * 2 + (lane >> 4)), b0, b1, b2, b3);
#pragma unroll
                            for (int m = 0; m < MG; ++m) {
                                mma_bf16(oacc[m][2 * dp], pa[m][ks][0], pa[m][ks][1], pa[m][ks][2],
                                         pa[m][ks][3], b0, b1);
                                mma_bf16(oacc[m][2 * dp + 1], pa[m][ks][0], pa[m][ks][1],
                                         pa[m][ks][2], pa[m][ks][3], b2, b3);
                            }
                        }
                    }
                }
#pragma unroll
                for (int m = 0; m < MG; ++m) {
                    const int r0 = (mg + m) * 16 + g, r1 = r0 + 8;
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) {
                        const int c = dh * 4 + nt;
                        if (r0 < T)
                            *reinterpret_cast<uint32_t *>(sq + swz(r0, c) + 4 * tq) =
                                pack_bf16x2(oacc[m][nt][0] * il[m][0], oacc[m][nt][1] * il[m][0]);
                        if (r1 < T)
                            *reinterpret_cast<uint32_t *>(sq + swz(r1, c) + 4 * tq) =
                                pack_bf16x2(oacc[m][nt][2] * il[m][1], oacc[m][nt][3] * il[m][1]);
                    }
                }
            }
        }
        __syncwarp();
        for (int r = rlane; r < T; r += 2)
            *reinterpret_cast<uint4 *>(a.o + base + r * tstride + cch * 8) =
                *reinterpret_cast<const uint4 *>(sq + swz(r, cch));
        __syncwarp();
    }
}

}  // namespace tp
}  // namespace va3d

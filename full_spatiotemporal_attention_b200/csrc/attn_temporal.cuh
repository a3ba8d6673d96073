// Temporal pass of factorised attention (handbook "How attention sees time":
// at each spatial position, attention along time over H'W' sequences of T'
// tokens).  Token (t, h, w) of a sequence sits at row t*H'W' + h*W' + w, so a
// position's T' rows are H'W' rows apart.
//
// The pass is HBM-bound (each position reads T' rows of Q, K, V and writes T'
// rows of O; its 4*T'^2*d FLOPs are small), so the design goal is streaming:
//  - persistent warps (up to 16 per SM, as many as shared memory holds), one
//    (batch*head, position) task at a time, rows fetched with 16-byte
//    cp.async (each row is 256 contiguous bytes); the other resident warps
//    compute while one waits for its rows;
//  - only the T' real rows are staged; m16n8k16 fragments that reach past
//    row T'-1 read row T'-1 again (their scores are masked or their outputs
//    dropped), so nothing is zero-filled;
//  - Q and K are turned by 3D RoPE in shared memory from the angle table and
//    stored as fp16 scaled by a power of two chosen per task from the largest
//    input magnitude: the QK^T product then carries 11 mantissa bits instead
//    of bf16's 8 (the temporal softmax has only T' terms, so its outputs are
//    O(1) and rounding the rotated operands would dominate the error), and the
//    exact power-of-two scale keeps any finite input in fp16 range;
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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

// Largest |x| over bf16 bit patterns, as a bit pattern (sign cleared); the
// ordering of such patterns follows the ordering of magnitudes.
__device__ __forceinline__ uint32_t absmax_bits(uint4 v, uint32_t m) {
    const uint32_t k = 0x7FFF7FFFu;
    uint32_t a = __vmaxu2(__vmaxu2(v.x & k, v.y & k), __vmaxu2(v.z & k, v.w & k));
    return max(m, max(a & 0xFFFFu, a >> 16));
}

// Power-of-two exponent s such that every rotated element, scaled by 2^s, is
// below 2^14: |x| < 2^(e-126) for a bf16 exponent field e, a rotation can
// grow one element by at most sqrt(2).  Clamped so the combined scale of two
// operands stays a normal float.
__device__ __forceinline__ int fp16_scale_exponent(uint32_t absmax_bits) {
    const int e = static_cast<int>((absmax_bits >> 7) & 0xFF);
    return max(-60, min(60, 139 - e));
}

__device__ __forceinline__ float pow2f(int s) {
    return __uint_as_float(static_cast<uint32_t>(127 + s) << 23);
}

template <int MAXT>
struct Cfg {
    static constexpr int kMaxWarps = 16;
    static constexpr int kSmemBudget = 208 * 1024;
};

// Shared memory per warp: (Q, K, V) with T rows of 256 bytes.
__host__ __device__ inline int temporal_warp_bytes(int T) { return 3 * T * 256; }

template <int MAXT>
__global__ void __launch_bounds__(Cfg<MAXT>::kMaxWarps * 32)
temporal_kernel(const __grid_constant__ TemporalArgs a) {
    constexpr int NP = MAXT / 16;   // pairs of n8 key tiles (and k16 steps over keys)
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int T = a.T;
    const int tensor_bytes = T * 256;
    const long long total = static_cast<long long>(a.BH) * a.HW;
    const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
    long long task = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (task >= total) return;   // the whole warp leaves together; no block barrier is used

    uint8_t *wbase = smem + warp * temporal_warp_bytes(T);
    const size_t tstride = static_cast<size_t>(a.HW) * 128;   // elements between frames

    auto row0 = [&](long long tk) -> size_t {   // element offset of frame 0 of a task
        const long long bh = tk / a.HW;
        const long long pos = tk - bh * a.HW;
        return (static_cast<size_t>(bh) * a.N + static_cast<size_t>(pos)) * 128;
    };
    auto issue = [&](long long tk, int) {
        const size_t base = row0(tk);
        const uint32_t s0 = smem_u32(wbase);
        for (int idx = lane; idx < T * 16; idx += 32) {
            const int r = idx >> 4, c = idx & 15;
            const uint32_t off = swz(r, c);
            const size_t g = base + r * tstride + c * 8;
            cp_async16(s0 + off, a.q + g);
            cp_async16(s0 + tensor_bytes + off, a.k + g);
            cp_async16(s0 + 2 * tensor_bytes + off, a.v + g);
        }
        cp_async_commit();
    };

    const int g = lane >> 2;   // fragment row
    const int tq = lane & 3;   // fragment column pair
    // In the RoPE and scale passes a lane always handles the same 16-byte
    // chunk (pairs 4c .. 4c+3) of rows (lane >> 4), (lane >> 4) + 2, ...
    const int cch = lane & 15;
    const int rlane = lane >> 4;
    uint8_t *sq = wbase;
    uint8_t *sk = sq + tensor_bytes;
    uint8_t *sv = sk + tensor_bytes;
    const uint32_t aq = smem_u32(sq), ak = smem_u32(sk), av = smem_u32(sv);
    for (; task < total; task += stride) {
        issue(task, 0);
        cp_async_wait<0>();
        __syncwarp();
        const long long bh = task / a.HW;
        const int pos = static_cast<int>(task - bh * a.HW);

        // ---- per-task fp16 scales for Q and K
        uint32_t mq = 0, mk = 0;
#pragma unroll 4
        for (int r = rlane; r < T; r += 2) {
            const uint32_t off = swz(r, cch);
            mq = absmax_bits(*reinterpret_cast<const uint4 *>(sq + off), mq);
            mk = absmax_bits(*reinterpret_cast<const uint4 *>(sk + off), mk);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mq = max(mq, __shfl_xor_sync(0xffffffffu, mq, o));
            mk = max(mk, __shfl_xor_sync(0xffffffffu, mk, o));
        }
        const int eq = fp16_scale_exponent(mq), ek = fp16_scale_exponent(mk);
        const float sq_f = pow2f(eq), sk_f = pow2f(ek);
        const float scale_log2 = a.scale_log2 * pow2f(-(eq + ek));

        // ---- rotate (RoPE) and convert Q and K to scaled fp16 in place.
        // Angles of h and w pairs are fixed for the task; t pairs vary by row.
        const int h = pos / a.rp.W;
        const int w = pos - h * a.rp.W;
        float2 cs_fixed[4];
        bool is_t[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int p = cch * 4 + e;
            is_t[e] = p < a.rp.pe_t;
            cs_fixed[e] = is_t[e] ? make_float2(1.f, 0.f) : a.rope_tab[table_index(a.rp, p, 0, h, w)];
        }
#pragma unroll 2
        for (int r = rlane; r < T; r += 2) {
            const uint32_t off = swz(r, cch);
            uint4 *pq = reinterpret_cast<uint4 *>(sq + off);
            uint4 *pk = reinterpret_cast<uint4 *>(sk + off);
            uint4 vq = *pq, vk = *pk;
            uint32_t *eqv = reinterpret_cast<uint32_t *>(&vq);
            uint32_t *ekv = reinterpret_cast<uint32_t *>(&vk);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 cs = is_t[e] ? a.rope_tab[r * a.rp.half_t + cch * 4 + e] : cs_fixed[e];
                const float2 x = unpack_bf16x2(eqv[e]);
                eqv[e] = pack_f16x2((x.x * cs.x - x.y * cs.y) * sq_f, (x.x * cs.y + x.y * cs.x) * sq_f);
                const float2 y = unpack_bf16x2(ekv[e]);
                if (a.rope_k)
                    ekv[e] = pack_f16x2((y.x * cs.x - y.y * cs.y) * sk_f, (y.x * cs.y + y.y * cs.x) * sk_f);
                else
                    ekv[e] = pack_f16x2(y.x * sk_f, y.y * sk_f);
            }
            *pq = vq;
            *pk = vk;
        }
        __syncwarp();

        const int tl = T - 1;
        for (int mt = 0; mt < NP; ++mt) {
            if (mt * 16 >= T) break;
            // ---- S = Q K^T for query rows mt*16 .. mt*16+15 (keys padded to NP*16)
            float sacc[2 * NP][4];
#pragma unroll
            for (int nt = 0; nt < 2 * NP; ++nt)
                sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
            const int qrow = min(mt * 16 + (lane & 15), tl);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(aq + swz(qrow, kk * 2 + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
                for (int np = 0; np < NP; ++np) {
                    if (np * 16 < T) {
                        uint32_t b0, b1, b2, b3;
                        const int krow = min(np * 16 + (lane & 7) + ((lane >> 4) << 3), tl);
                        ldsm_x4(ak + swz(krow, kk * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
                        mma_f16(sacc[2 * np], a0, a1, a2, a3, b0, b1);
                        mma_f16(sacc[2 * np + 1], a0, a1, a2, a3, b2, b3);
                    }
                }
            }
            // ---- softmax over the T keys (rows g and g+8 of the m-tile)
            float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2 * NP; ++nt) {
                const int c0 = nt * 8 + 2 * tq;
                if (c0 >= T) { sacc[nt][0] = -INFINITY; sacc[nt][2] = -INFINITY; }
                if (c0 + 1 >= T) { sacc[nt][1] = -INFINITY; sacc[nt][3] = -INFINITY; }
                m0 = fmax3(m0, sacc[nt][0], sacc[nt][1]);
                m1 = fmax3(m1, sacc[nt][2], sacc[nt][3]);
            }
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
            const float nm0 = -m0 * scale_log2, nm1 = -m1 * scale_log2;
            float l0 = 0.f, l1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2 * NP; ++nt) {
                sacc[nt][0] = ex2(fmaf(sacc[nt][0], scale_log2, nm0));
                sacc[nt][1] = ex2(fmaf(sacc[nt][1], scale_log2, nm0));
                sacc[nt][2] = ex2(fmaf(sacc[nt][2], scale_log2, nm1));
                sacc[nt][3] = ex2(fmaf(sacc[nt][3], scale_log2, nm1));
                l0 += sacc[nt][0] + sacc[nt][1];
                l1 += sacc[nt][2] + sacc[nt][3];
            }
            l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
            l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
            const float il0 = 1.f / l0, il1 = 1.f / l1;
            // P as bf16 A fragments, k = key index
            uint32_t pa[NP][4];
#pragma unroll
            for (int ks = 0; ks < NP; ++ks) {
                pa[ks][0] = pack_bf16x2(sacc[2 * ks][0], sacc[2 * ks][1]);
                pa[ks][1] = pack_bf16x2(sacc[2 * ks][2], sacc[2 * ks][3]);
                pa[ks][2] = pack_bf16x2(sacc[2 * ks + 1][0], sacc[2 * ks + 1][1]);
                pa[ks][3] = pack_bf16x2(sacc[2 * ks + 1][2], sacc[2 * ks + 1][3]);
            }
            __syncwarp();
            // ---- O = P V, 64 output columns at a time, staged into this m-tile's Q rows
#pragma unroll
            for (int dh = 0; dh < 2; ++dh) {
                float oacc[8][4];
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
                    oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
#pragma unroll
                for (int ks = 0; ks < NP; ++ks) {
                    if (ks * 16 < T) {
                        const int vrow = min(ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), tl);
#pragma unroll
                        for (int dp = 0; dp < 4; ++dp) {
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4_t(av + swz(vrow, dh * 8 + dp * 2 + (lane >> 4)), b0, b1, b2, b3);
                            mma_bf16(oacc[2 * dp], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b0, b1);
                            mma_bf16(oacc[2 * dp + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b2, b3);
                        }
                    }
                }
                const int r0 = mt * 16 + g, r1 = r0 + 8;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    const int c = dh * 8 + nt;
                    if (r0 < T)
                        *reinterpret_cast<uint32_t *>(sq + swz(r0, c) + 4 * tq) =
                            pack_bf16x2(oacc[nt][0] * il0, oacc[nt][1] * il0);
                    if (r1 < T)
                        *reinterpret_cast<uint32_t *>(sq + swz(r1, c) + 4 * tq) =
                            pack_bf16x2(oacc[nt][2] * il1, oacc[nt][3] * il1);
                }
            }
        }
        __syncwarp();
        const size_t base = row0(task);
        for (int idx = lane; idx < T * 16; idx += 32) {
            const int r = idx >> 4, c = idx & 15;
            const uint4 v = *reinterpret_cast<const uint4 *>(sq + swz(r, c));
            *reinterpret_cast<uint4 *>(a.o + base + r * tstride + c * 8) = v;
        }
        __syncwarp();
    }
}

}  // namespace tp
}  // namespace va3d

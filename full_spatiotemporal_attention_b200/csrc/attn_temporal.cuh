// Temporal pass of factorised attention (handbook "How attention sees time":
// at each spatial position, attention along time over H'W' sequences of T'
// tokens).  Token (t, h, w) of a sequence sits at row t*H'W' + h*W' + w, so a
// position's T' rows are H'W' rows apart.
//
// The pass is HBM-bound (each position reads T' rows of Q, K, V and writes T'
// rows of O; the 4*T'^2*d FLOPs are small), so the design goal is streaming:
// one warp per (batch*head, position), rows fetched with 16-byte cp.async
// (each row is 256 contiguous bytes), Q turned by 3D RoPE in shared memory
// from the angle table, S = Q K^T and O = P V on the m16n8k16 bf16 tensor-core
// path with fp32 accumulation, and O staged through shared memory so the
// global stores are 16-byte and row-contiguous.  Sequences are padded to
// MAXT rows (32 or 64); padded keys are masked, padded rows are not stored.
#pragma once

#include "ptx.cuh"
#include "rope.cuh"

namespace va3d {
namespace tp {

struct TemporalArgs {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k;    // rotated keys
    const __nv_bfloat16 *v;
    __nv_bfloat16 *o;
    int N;                     // tokens per sequence (T*HW)
    int T;                     // frames T'
    int HW;                    // positions per frame H'W'
    int BH;                    // batch * heads
    float scale_log2;
    int rope_q;
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

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
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

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int MAXT>
struct Cfg {
    static constexpr int kWarps = MAXT <= 32 ? 4 : 2;
    static constexpr int kTensorBytes = MAXT * 256;
    static constexpr int kWarpBytes = 3 * kTensorBytes;
    static constexpr int kSmemBytes = kWarps * kWarpBytes;
};

template <int MAXT>
__global__ void __launch_bounds__(Cfg<MAXT>::kWarps * 32)
temporal_kernel(const __grid_constant__ TemporalArgs a) {
    constexpr int NT = MAXT / 8;    // n8 tiles of keys
    constexpr int KT = MAXT / 16;   // k16 steps over keys in PV
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long task = static_cast<long long>(blockIdx.x) * Cfg<MAXT>::kWarps + warp;
    if (task >= static_cast<long long>(a.BH) * a.HW) return;   // whole warp leaves together
    const int bh = static_cast<int>(task / a.HW);
    const int pos = static_cast<int>(task - static_cast<long long>(bh) * a.HW);
    const int T = a.T;

    uint8_t *sq = smem + warp * Cfg<MAXT>::kWarpBytes;
    uint8_t *sk = sq + Cfg<MAXT>::kTensorBytes;
    uint8_t *sv = sk + Cfg<MAXT>::kTensorBytes;
    const uint32_t aq = smem_u32(sq), ak = smem_u32(sk), av = smem_u32(sv);

    // element offset of (row t = 0) of this position; row t adds t*HW*128
    const size_t base = (static_cast<size_t>(bh) * a.N + pos) * 128;
    const size_t tstride = static_cast<size_t>(a.HW) * 128;

    for (int idx = lane; idx < MAXT * 16; idx += 32) {
        const int r = idx >> 4, c = idx & 15;
        const uint32_t off = swz(r, c);
        if (r < T) {
            const size_t g = base + r * tstride + c * 8;
            cp_async16(aq + off, a.q + g);
            cp_async16(ak + off, a.k + g);
            cp_async16(av + off, a.v + g);
        } else {
            const uint4 z = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sq + off) = z;
            *reinterpret_cast<uint4 *>(sk + off) = z;
            *reinterpret_cast<uint4 *>(sv + off) = z;
        }
    }
    cp_async_wait_all();
    __syncwarp();

    if (a.rope_q) {
        const int h = pos / a.rp.W;
        const int w = pos - h * a.rp.W;
        for (int idx = lane; idx < T * 16; idx += 32) {
            const int r = idx >> 4, c = idx & 15;
            uint4 *p = reinterpret_cast<uint4 *>(sq + swz(r, c));
            uint4 v = *p;
            const int p0 = c * 4;
            v.x = rotate_pair(v.x, a.rope_tab[table_index(a.rp, p0 + 0, r, h, w)]);
            v.y = rotate_pair(v.y, a.rope_tab[table_index(a.rp, p0 + 1, r, h, w)]);
            v.z = rotate_pair(v.z, a.rope_tab[table_index(a.rp, p0 + 2, r, h, w)]);
            v.w = rotate_pair(v.w, a.rope_tab[table_index(a.rp, p0 + 3, r, h, w)]);
            *p = v;
        }
        __syncwarp();
    }

    const int g = lane >> 2;        // fragment row
    const int tq = lane & 3;        // fragment column pair
    for (int mt = 0; mt < KT; ++mt) {
        if (mt * 16 >= T) break;
        // ---- S = Q K^T for query rows mt*16 .. mt*16+15
        float sacc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(aq + swz(mt * 16 + (lane & 15), kk * 2 + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(ak + swz(np * 16 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)),
                        b0, b1, b2, b3);
                mma16816(sacc[2 * np], a0, a1, a2, a3, b0, b1);
                mma16816(sacc[2 * np + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        // ---- softmax over the T valid keys (rows g and g+8 of the m-tile)
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int c0 = nt * 8 + 2 * tq;
            if (c0 >= T) { sacc[nt][0] = -INFINITY; sacc[nt][2] = -INFINITY; }
            if (c0 + 1 >= T) { sacc[nt][1] = -INFINITY; sacc[nt][3] = -INFINITY; }
            m0 = fmaxf(m0, fmaxf(sacc[nt][0], sacc[nt][1]));
            m1 = fmaxf(m1, fmaxf(sacc[nt][2], sacc[nt][3]));
        }
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
        const float nm0 = -m0 * a.scale_log2, nm1 = -m1 * a.scale_log2;
        float l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            sacc[nt][0] = ex2(fmaf(sacc[nt][0], a.scale_log2, nm0));
            sacc[nt][1] = ex2(fmaf(sacc[nt][1], a.scale_log2, nm0));
            sacc[nt][2] = ex2(fmaf(sacc[nt][2], a.scale_log2, nm1));
            sacc[nt][3] = ex2(fmaf(sacc[nt][3], a.scale_log2, nm1));
            l0 += sacc[nt][0] + sacc[nt][1];
            l1 += sacc[nt][2] + sacc[nt][3];
        }
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        const float il0 = 1.f / l0, il1 = 1.f / l1;
        // P as A fragments (bf16), k = key index
        uint32_t pa[KT][4];
#pragma unroll
        for (int ks = 0; ks < KT; ++ks) {
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
            for (int nt = 0; nt < 8; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KT; ++ks) {
#pragma unroll
                for (int dp = 0; dp < 4; ++dp) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(av + swz(ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3),
                                       dh * 8 + dp * 2 + (lane >> 4)),
                              b0, b1, b2, b3);
                    mma16816(oacc[2 * dp], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b0, b1);
                    mma16816(oacc[2 * dp + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b2, b3);
                }
            }
            const int r0 = mt * 16 + g, r1 = r0 + 8;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int c = dh * 8 + nt;
                *reinterpret_cast<uint32_t *>(sq + swz(r0, c) + 4 * tq) =
                    pack_bf16x2(oacc[nt][0] * il0, oacc[nt][1] * il0);
                *reinterpret_cast<uint32_t *>(sq + swz(r1, c) + 4 * tq) =
                    pack_bf16x2(oacc[nt][2] * il1, oacc[nt][3] * il1);
            }
        }
    }
    __syncwarp();
    for (int idx = lane; idx < T * 16; idx += 32) {
        const int r = idx >> 4, c = idx & 15;
        const uint4 v = *reinterpret_cast<const uint4 *>(sq + swz(r, c));
        *reinterpret_cast<uint4 *>(a.o + base + r * tstride + c * 8) = v;
    }
}

}  // namespace tp
}  // namespace va3d

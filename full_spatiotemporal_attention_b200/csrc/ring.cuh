// Ring context parallelism: key/value blocks travel around the ranks while
// each rank attends its own query slice to every block in turn, merging the
// partial outputs by their log-sum-exp.  It needs no head split, so it
// serves more ranks than heads (the anthology record on full 3D attention,
// sota-390, names ring and Ulysses context parallelism as what long videos
// turn to).
//
// Rank r holds tokens [r*n_loc, (r+1)*n_loc) of every head.  Positions are
// absolute (handbook "A video model's architecture", section "Position: RoPE
// in three dimensions"), so the load kernel turns this rank's Q and K at
// their global positions once; every block product afterwards is a plain
// softmax(q k^T) v over one block of keys (the cross-attention form of the
// attention kernel, with its LSE).  For block outputs (o_1, l_1) and
// (o_2, l_2) of the same query row, with m = max(l_1, l_2),
//   l = m + log(e^(l_1 - m) + e^(l_2 - m)),
//   o = (e^(l_1 - m) o_1 + e^(l_2 - m) o_2) / (e^(l_1 - m) + e^(l_2 - m)),
// which is the softmax over the union of the two key sets.
//
// Every rank owns one region, mapped into its ring neighbours:
//   [ header: u64 counters (full, free) | K0 | V0 | K1 | V1 ]
// each block buffer [B, heads, n_loc, 128] bf16.  At step s a rank attends
// buffer s % 2 and copies it into the next rank's buffer (s + 1) % 2 (blocks
// signal the next rank's `full` counter as in the Ulysses exchange); after
// its product it bumps the previous rank's `free` counter, which the
// previous rank waits on before overwriting this rank's buffer again.
#pragma once

#include "ulysses.cuh"

namespace va3d {
namespace ring {

constexpr size_t kHeaderBytes = 256;
enum Counter { kFull = 0, kFree = 1 };

struct Layout {
    size_t k[2], v[2];
    size_t bytes;
};

inline Layout region_layout(int B, int heads, int N, int world) {
    const size_t blk = static_cast<size_t>(B) * heads * (N / world) * 256;
    Layout l;
    l.k[0] = kHeaderBytes;
    l.v[0] = l.k[0] + blk;
    l.k[1] = l.v[0] + blk;
    l.v[1] = l.k[1] + blk;
    l.bytes = l.v[1] + blk;
    return l;
}

struct LoadArgs {
    const uint4 *q, *k, *v;   // local slice [B*heads, n_loc, 128]
    uint4 *q_rot, *k0, *v0;   // this rank's turned queries and block buffer 0
    long long rows;           // B * heads
    int n_loc, offset;        // tokens per rank, global index of the first
    int rope_q, rope_k;
};

// Thread (n, c): local token n, chunk c, over every (batch, head) row; the
// angles are computed once per token (as in the key pre-pass).
__global__ void __launch_bounds__(cp::kCopyThreads)
ring_load_kernel(const __grid_constant__ LoadArgs a, const __grid_constant__ RopeParams rp) {
    const long long total = static_cast<long long>(a.n_loc) * 16;
    const size_t row = static_cast<size_t>(a.n_loc) * 16;
    for (long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; gid < total;
         gid += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int n = static_cast<int>(gid >> 4);
        const int c = static_cast<int>(gid & 15);
        const int g = a.offset + n;
        const bool video = g < rp.n_video;
        float2 cs[4];
        if (video) {
            const int t = g / rp.HW;
            const int rem = g - t * rp.HW;
            const int h = rem / rp.W;
            const int w = rem - h * rp.W;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int p = c * 4 + e;
                cs[e] = rope_cs(rp.inv_freq[p], pair_pos(rp, p, t, h, w));
            }
        }
        for (long long r0 = 0; r0 < a.rows; r0 += cp::kScatterRows) {
            uint4 xq[cp::kScatterRows], xk[cp::kScatterRows], xv[cp::kScatterRows];
#pragma unroll
            for (int u = 0; u < cp::kScatterRows; ++u) {
                if (r0 + u < a.rows) {
                    const size_t s = static_cast<size_t>(r0 + u) * row + gid;
                    xq[u] = a.q[s];
                    xk[u] = a.k[s];
                    xv[u] = a.v[s];
                }
            }
#pragma unroll
            for (int u = 0; u < cp::kScatterRows; ++u) {
                if (r0 + u < a.rows) {
                    if (video && a.rope_q) {
                        xq[u].x = rotate_pair(xq[u].x, cs[0]);
                        xq[u].y = rotate_pair(xq[u].y, cs[1]);
                        xq[u].z = rotate_pair(xq[u].z, cs[2]);
                        xq[u].w = rotate_pair(xq[u].w, cs[3]);
                    }
                    if (video && a.rope_k) {
                        xk[u].x = rotate_pair(xk[u].x, cs[0]);
                        xk[u].y = rotate_pair(xk[u].y, cs[1]);
                        xk[u].z = rotate_pair(xk[u].z, cs[2]);
                        xk[u].w = rotate_pair(xk[u].w, cs[3]);
                    }
                    const size_t s = static_cast<size_t>(r0 + u) * row + gid;
                    a.q_rot[s] = xq[u];
                    a.k0[s] = xk[u];
                    a.v0[s] = xv[u];
                }
            }
        }
    }
}

// Copy this rank's K and V block buffer to the next rank's other buffer,
// then signal the next rank's `full` counter (one per block of the grid).
__global__ void __launch_bounds__(cp::kCopyThreads)
ring_pass_kernel(const uint4 *k_src, const uint4 *v_src, uint4 *k_dst, uint4 *v_dst, long long chunks,
                 uint8_t *dst_region) {
    for (long long i0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < chunks;
         i0 += static_cast<long long>(gridDim.x) * blockDim.x * cp::kScatterRows) {
        uint4 xk[cp::kScatterRows], xv[cp::kScatterRows];
        const long long step = static_cast<long long>(gridDim.x) * blockDim.x;
#pragma unroll
        for (int u = 0; u < cp::kScatterRows; ++u) {
            const long long i = i0 + u * step;
            if (i < chunks) {
                xk[u] = k_src[i];
                xv[u] = v_src[i];
            }
        }
#pragma unroll
        for (int u = 0; u < cp::kScatterRows; ++u) {
            const long long i = i0 + u * step;
            if (i < chunks) {
                k_dst[i] = xk[u];
                v_dst[i] = xv[u];
            }
        }
    }
    uint8_t *regions[1] = {dst_region};
    cp::signal_peers(regions, 1, kFull);
}

// This rank has finished reading its current buffer: one increment of the
// previous rank's `free` counter.  The product that read the buffer is
// complete before this kernel starts (stream order), so no fence is needed
// for the reads themselves.
__global__ void ring_free_kernel(uint8_t *prev_region) {
    if (threadIdx.x == 0)
        atomicAdd_system(reinterpret_cast<unsigned long long *>(prev_region) + kFree, 1ull);
}

// Merge one block's output into the running fp32 accumulator.  Thread
// (row, 8-element chunk).  lse_in is the accumulator's LSE before this
// block, lse_out after it (two buffers, so no thread reads a value another
// thread of the same row has already replaced).  `first`: the accumulator
// starts as this block.  `out` (nullable): also write the merged output as
// bf16 (the last block).
__global__ void __launch_bounds__(256)
ring_merge_kernel(const uint4 *o_blk, const float *lse_blk, float4 *acc, const float *lse_in,
                  float *lse_out, uint4 *out, long long rows, int first) {
    const long long total = rows * 16;
    for (long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; gid < total;
         gid += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long r = gid >> 4;
        const float2 o01 = unpack_bf16x2(o_blk[gid].x), o23 = unpack_bf16x2(o_blk[gid].y);
        const float2 o45 = unpack_bf16x2(o_blk[gid].z), o67 = unpack_bf16x2(o_blk[gid].w);
        float x[8] = {o01.x, o01.y, o23.x, o23.y, o45.x, o45.y, o67.x, o67.y};
        const float lb = lse_blk[r];
        float l = lb;
        if (!first) {
            const float la = lse_in[r];
            const float m = fmaxf(la, lb);
            const float wa = expf(la - m), wb = expf(lb - m);
            const float inv = 1.0f / (wa + wb);
            const float4 a0 = acc[2 * gid], a1 = acc[2 * gid + 1];
            const float y[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = (wa * y[e] + wb * x[e]) * inv;
            l = m + logf(wa + wb);
        }
        acc[2 * gid] = make_float4(x[0], x[1], x[2], x[3]);
        acc[2 * gid + 1] = make_float4(x[4], x[5], x[6], x[7]);
        if ((gid & 15) == 0) lse_out[r] = l;
        if (out != nullptr)
            out[gid] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                  pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
    }
}

}  // namespace ring
}  // namespace va3d

// 3D RoPE on B200: angle table and the HBM-bound rotation kernel.
//
// Token n of a sequence is a video token when n < T'H'W', at
// (t, h, w) = (n / H'W', (n / W') % H', n % W'); text tokens (n >= T'H'W')
// are not rotated.  The head dim is split into the t, h and w ranges
// [0, d_t), [d_t, d_t+d_h), [d_t+d_h, 128); pair p = (2p, 2p+1) belongs to
// one range and turns by pos_axis * inv_freq[p], with
// inv_freq = theta^(-2j/d_axis) for its index j inside the range (handbook
// "A video model's architecture", section "Position: RoPE in three
// dimensions"; CogVideoX guide section 3, block-diagonal R_3D).
#pragma once

#include "ptx.cuh"

namespace va3d {

struct RopeParams {
    int T, H, W;
    int HW;
    int n_video;               // T*H*W; tokens at or past this index are text
    int pe_t, pe_h;            // pairs [0,pe_t) turn with t, [pe_t,pe_h) with h, the rest with w
    int half_t, half_h, half_w;  // pairs per axis (d_axis / 2)
    int tab_h, tab_w;          // table offsets (entries) of the h and w sections; t is at 0
                               // (each section pair-major: entry (j, pos) at j * extent + pos)
    int tab_entries;           // T*half_t + H*half_h + W*half_w
    float inv_freq[64];        // per pair; computed on the host in fp64, rounded to fp32
};

// Axis position of pair p for a token at (t, h, w).
__device__ __forceinline__ int pair_pos(const RopeParams &rp, int p, int t, int h, int w) {
    return p < rp.pe_t ? t : (p < rp.pe_h ? h : w);
}

// cos and sin of pair p's angle at axis position `pos` (fp32, accurate sincosf).
__device__ __forceinline__ float2 rope_cs(float inv_freq, int pos) {
    float s, c;
    sincosf(static_cast<float>(pos) * inv_freq, &s, &c);
    return make_float2(c, s);
}

// Table entry of pair p for a token at (t, h, w) (same layout as
// rope_table_kernel).  Pair-major sections: threads that hold consecutive
// tokens (consecutive w) read consecutive entries for the same pair.
__device__ __forceinline__ int table_index(const RopeParams &rp, int p, int t, int h, int w) {
    if (p < rp.pe_t) return p * rp.T + t;
    if (p < rp.pe_h) return rp.tab_h + (p - rp.pe_t) * rp.H + h;
    return rp.tab_w + (p - rp.pe_h) * rp.W + w;
}

// (x0, x1) -> (x0 c - x1 s, x0 s + x1 c) on one packed bf16 pair.
__device__ __forceinline__ uint32_t rotate_pair(uint32_t packed, float2 cs) {
    float2 f = unpack_bf16x2(packed);
    float y0 = f.x * cs.x - f.y * cs.y;
    float y1 = f.x * cs.y + f.y * cs.x;
    return pack_bf16x2(y0, y1);
}

// Build the cos/sin table for a grid: entries (j, t) at j*T + t, then
// (j, h) at tab_h + j*H + h, then (j, w) at tab_w + j*W + w.
// It also clears `n_zero` ints at `zero` (per-call counters of the attention
// kernel that follows on the same stream).
__global__ void rope_table_kernel(float2 *__restrict__ tab, int *__restrict__ zero, int n_zero,
                                  const __grid_constant__ RopeParams rp) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n_zero; e += gridDim.x * blockDim.x)
        zero[e] = 0;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < rp.tab_entries;
         e += gridDim.x * blockDim.x) {
        int p, pos;
        if (e < rp.tab_h) {
            p = e / rp.T;
            pos = e - p * rp.T;
        } else if (e < rp.tab_w) {
            const int r = e - rp.tab_h;
            const int j = r / rp.H;
            pos = r - j * rp.H;
            p = rp.pe_t + j;
        } else {
            const int r = e - rp.tab_w;
            const int j = r / rp.W;
            pos = r - j * rp.W;
            p = rp.pe_h + j;
        }
        tab[e] = rope_cs(rp.inv_freq[p], pos);
    }
}

// y = RoPE(x) for [BH, N, 128] bf16.  One thread per (token, 16-byte chunk)
// computes the four angles of its chunk once and applies them to the chunk
// in every (batch, head) row, four rows in flight at a time.  x may equal y.
// It also clears `n_zero` ints at `zero` (the split-tail counters of the
// attention launch that follows on the same stream).
constexpr int kRopeThreads = 256;

__global__ void __launch_bounds__(kRopeThreads)
rope_apply_kernel(const uint4 *x, uint4 *y, long long N, int BH,
                  const __grid_constant__ RopeParams rp, int *zero, int n_zero) {
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gid < n_zero) zero[gid] = 0;
    if (gid >= N * 16) return;
    const int n = static_cast<int>(gid >> 4);
    const int c = static_cast<int>(gid & 15);
    const bool video = n < rp.n_video;

    float2 cs[4];
    if (video) {
        const int t = n / rp.HW;
        const int rem = n - t * rp.HW;
        const int h = rem / rp.W;
        const int w = rem - h * rp.W;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int p = c * 4 + e;
            cs[e] = rope_cs(rp.inv_freq[p], pair_pos(rp, p, t, h, w));
        }
    }

    const size_t stride = static_cast<size_t>(N) * 16;   // uint4 per (batch, head) row block
    size_t idx = static_cast<size_t>(gid);
    int bh = 0;
    for (; bh + 4 <= BH; bh += 4) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = x[idx + static_cast<size_t>(bh + u) * stride];
        if (video) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                v[u].x = rotate_pair(v[u].x, cs[0]);
                v[u].y = rotate_pair(v[u].y, cs[1]);
                v[u].z = rotate_pair(v[u].z, cs[2]);
                v[u].w = rotate_pair(v[u].w, cs[3]);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) y[idx + static_cast<size_t>(bh + u) * stride] = v[u];
    }
    for (; bh < BH; ++bh) {
        uint4 v = x[idx + static_cast<size_t>(bh) * stride];
        if (video) {
            v.x = rotate_pair(v.x, cs[0]);
            v.y = rotate_pair(v.y, cs[1]);
            v.z = rotate_pair(v.z, cs[2]);
            v.w = rotate_pair(v.w, cs[3]);
        }
        y[idx + static_cast<size_t>(bh) * stride] = v;
    }
}

}  // namespace va3d

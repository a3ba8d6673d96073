// Ulysses context parallelism: sequence shards <-> head shards over peer
// memory (NVLink / NVSwitch), with the key RoPE fused into the exchange.
//
// Rank r of P holds the contiguous token slice [r*n_loc, (r+1)*n_loc) of
// every head, n_loc = N / P.  Full attention needs whole sequences, so the
// heads are regrouped: rank j receives heads [j*hpw, (j+1)*hpw) (hpw =
// heads / P) for all N tokens, runs attention on them, and sends each
// token slice of its output back to the rank that owns it.  RoPE needs no
// exchange of its own because positions are absolute (handbook "A video
// model's architecture", section "Position: RoPE in three dimensions": each
// rank holds a contiguous token segment and knows its tokens' global
// coordinates), so keys are turned on the way out.  The anthology record on
// full 3D attention (sota-390) names Ulysses and ring context parallelism as
// what long videos turn to.
//
// Every rank owns one region, mapped into every other rank's address space:
//   [ header: u64 counters (scatter, gather) | Qh | Kh | Vh | O shard ]
// Qh, Kh, Vh are [B, hpw, N, 128] bf16 (this rank's heads, all tokens) and
// the O shard is [B, heads, n_loc, 128] bf16 (all heads, this rank's tokens).
//
// Both copy kernels write straight into the peers' regions with 16-byte
// stores, then every thread fences at system scope and one thread per block
// adds 1 to each peer's counter for the phase.  A peer knows its region is
// complete for epoch e when its counter reaches e * P * blocks, which the
// bounded wait kernel checks before anything reads the region.
#pragma once

#include "rope.cuh"

namespace va3d {
namespace cp {

constexpr int kMaxWorld = 8;          // ranks of one NVSwitch node
constexpr int kCopyThreads = 256;
constexpr int kMaxCopyBlocks = 1024;  // fixed cap: the same grid on every rank
constexpr size_t kHeaderBytes = 256;
constexpr int kScatterRows = 2;       // (batch, head) rows whose loads are in flight together
constexpr int kGatherRows = 8;

enum Phase { kScatter = 0, kGather = 1 };

struct Layout {
    size_t q, k, v, o;  // byte offsets of Qh, Kh, Vh, O shard inside a region
    size_t bytes;       // whole region
};

inline Layout region_layout(int B, int heads, int N, int world) {
    const size_t head_shard = static_cast<size_t>(B) * (heads / world) * N * 256;
    const size_t seq_shard = static_cast<size_t>(B) * heads * (N / world) * 256;
    Layout l;
    l.q = kHeaderBytes;
    l.k = l.q + head_shard;
    l.v = l.k + head_shard;
    l.o = l.v + head_shard;
    l.bytes = l.o + seq_shard;
    return l;
}

// Blocks of a copy kernel over `rows` token rows (16 chunks each).
inline int copy_blocks(long long rows) {
    const long long need = (rows * 16 + kCopyThreads - 1) / kCopyThreads;
    return static_cast<int>(need < kMaxCopyBlocks ? need : kMaxCopyBlocks);
}

struct ScatterArgs {
    const uint4 *q, *k, *v;       // local [B, heads, n_loc, 128]
    uint8_t *region[kMaxWorld];   // every rank's region (own included)
    size_t off_q, off_k, off_v;
    int world, rank, B, heads, hpw, N, n_loc;
    int rotate_k;                 // 1: turn k by its global positions here
};

struct GatherArgs {
    const uint4 *o;               // local [B, hpw, N, 128] (this rank's heads)
    uint8_t *region[kMaxWorld];
    size_t off_o;
    int world, rank, B, heads, hpw, N, n_loc;
};

// Every thread of the block has made its stores: the barrier orders them
// before thread 0's system-scope fence, which (fences being cumulative)
// makes them visible everywhere before thread 0 bumps each peer's counter
// for this phase (the pattern of a grid-wide barrier, at system scope).
__device__ __forceinline__ void signal_peers(uint8_t *const *region, int world, int phase) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence_system();
        for (int j = 0; j < world; ++j)
            atomicAdd_system(reinterpret_cast<unsigned long long *>(region[j]) + phase, 1ull);
    }
}

// Thread (n, c): local token n, 16-byte chunk c (pairs 4c..4c+3), over every
// (batch, head) row.  Rows of head h go to rank h / hpw at token rank*n_loc+n.
__global__ void __launch_bounds__(kCopyThreads)
ulysses_scatter_kernel(const __grid_constant__ ScatterArgs a, const __grid_constant__ RopeParams rp) {
    const long long total = static_cast<long long>(a.n_loc) * 16;
    const size_t src_row = static_cast<size_t>(a.n_loc) * 16;   // uint4 per local (b, h) block
    const size_t dst_row = static_cast<size_t>(a.N) * 16;       // uint4 per remote (b, h') block
    for (long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; gid < total;
         gid += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int n = static_cast<int>(gid >> 4);
        const int c = static_cast<int>(gid & 15);
        const int g = a.rank * a.n_loc + n;   // global token index
        const bool turn = a.rotate_k && g < rp.n_video;
        float2 cs[4];
        if (turn) {
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
        // (batch, head) rows kScatterRows at a time: all their loads are issued
        // before any store (the stores may alias the sources as far as the
        // compiler knows, so it would not hoist the next loads itself)
        const int rows = a.B * a.heads;
        for (int r0 = 0; r0 < rows; r0 += kScatterRows) {
            uint4 xq[kScatterRows], xk[kScatterRows], xv[kScatterRows];
#pragma unroll
            for (int u = 0; u < kScatterRows; ++u) {
                if (r0 + u < rows) {
                    const size_t s = static_cast<size_t>(r0 + u) * src_row + gid;
                    xq[u] = a.q[s];
                    xk[u] = a.k[s];
                    xv[u] = a.v[s];
                }
            }
#pragma unroll
            for (int u = 0; u < kScatterRows; ++u) {
                if (r0 + u < rows) {
                    if (turn) {
                        xk[u].x = rotate_pair(xk[u].x, cs[0]);
                        xk[u].y = rotate_pair(xk[u].y, cs[1]);
                        xk[u].z = rotate_pair(xk[u].z, cs[2]);
                        xk[u].w = rotate_pair(xk[u].w, cs[3]);
                    }
                    const int b = (r0 + u) / a.heads;
                    const int h = r0 + u - b * a.heads;
                    const int j = h / a.hpw;
                    const size_t d = (static_cast<size_t>(b) * a.hpw + (h - j * a.hpw)) * dst_row +
                                     static_cast<size_t>(g) * 16 + c;
                    uint8_t *base = a.region[j];
                    reinterpret_cast<uint4 *>(base + a.off_q)[d] = xq[u];
                    reinterpret_cast<uint4 *>(base + a.off_k)[d] = xk[u];
                    reinterpret_cast<uint4 *>(base + a.off_v)[d] = xv[u];
                }
            }
        }
    }
    signal_peers(a.region, a.world, kScatter);
}

// Thread (g, c): global token g, chunk c, over this rank's (batch, head)
// rows; token g goes to rank g / n_loc, head rank*hpw + h'.
__global__ void __launch_bounds__(kCopyThreads) ulysses_gather_kernel(const __grid_constant__ GatherArgs a) {
    const long long total = static_cast<long long>(a.N) * 16;
    const size_t src_row = static_cast<size_t>(a.N) * 16;
    const size_t dst_row = static_cast<size_t>(a.n_loc) * 16;
    for (long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; gid < total;
         gid += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int g = static_cast<int>(gid >> 4);
        const int c = static_cast<int>(gid & 15);
        const int j = g / a.n_loc;
        const int n = g - j * a.n_loc;
        uint4 *dst = reinterpret_cast<uint4 *>(a.region[j] + a.off_o);
        const int rows = a.B * a.hpw;
        for (int r0 = 0; r0 < rows; r0 += kGatherRows) {
            uint4 x[kGatherRows];
#pragma unroll
            for (int u = 0; u < kGatherRows; ++u)
                if (r0 + u < rows) x[u] = a.o[static_cast<size_t>(r0 + u) * src_row + gid];
#pragma unroll
            for (int u = 0; u < kGatherRows; ++u) {
                if (r0 + u < rows) {
                    const int b = (r0 + u) / a.hpw;
                    const int h = r0 + u - b * a.hpw;
                    dst[(static_cast<size_t>(b) * a.heads + a.rank * a.hpw + h) * dst_row +
                        static_cast<size_t>(n) * 16 + c] = x[u];
                }
            }
        }
    }
    signal_peers(a.region, a.world, kGather);
}

__device__ __forceinline__ unsigned long long ld_acquire_sys(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Wait (bounded by kWaitLimitNs) until this rank's counter for `phase`
// reaches `expected`; on expiry record VA3D_DEVERR_TIMEOUT_PEER and return.
__global__ void ulysses_wait_kernel(const unsigned long long *counters, int phase,
                                    unsigned long long expected) {
    if (threadIdx.x != 0) return;
    const unsigned long long *p = counters + phase;
    if (ld_acquire_sys(p) >= expected) return;
    const unsigned long long t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (ld_acquire_sys(p) >= expected) return;
        if ((it & 63u) == 0u && global_ns() - t0 > kWaitLimitNs) {
            atomicCAS(&g_device_error, 0, VA3D_DEVERR_TIMEOUT_PEER);
            return;
        }
        __nanosleep(200);
    }
}

}  // namespace cp
}  // namespace va3d

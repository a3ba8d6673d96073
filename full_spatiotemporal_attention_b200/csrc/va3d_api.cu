// C ABI of libva3d.so: argument checks, tensor-map construction and kernel
// launches.  The whole library is one translation unit (the kernels live in
// the headers included below) so the device error word is shared by every
// kernel.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "va3d.h"
#include "ptx.cuh"
#include "rope.cuh"
#include "attn_sm100.cuh"
#include "attn_temporal.cuh"
#include "attn_temporal_tc.cuh"
#include "selftest.cuh"
#include "ulysses.cuh"
#include "ring.cuh"

using namespace va3d;

namespace {

constexpr int kHeadDim = 128;
constexpr double kLog2e = 1.4426950408889634;

// Host-side NVTX range over one entry point (header-only NVTX v3: without a
// profiler attached the calls return at once and nothing is linked).
struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange &) = delete;
    TraceRange &operator=(const TraceRange &) = delete;
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int check_grid(const va3d_grid_t *g, int N, int head_dim) {
    if (g == nullptr) return VA3D_ERR_INVALID;
    if (g->T < 1 || g->H < 1 || g->W < 1 || g->n_text < 0) return VA3D_ERR_INVALID;
    if (g->d_t < 0 || g->d_h < 0 || g->d_w < 0) return VA3D_ERR_INVALID;
    if ((g->d_t | g->d_h | g->d_w) & 1) return VA3D_ERR_INVALID;
    if (g->d_t + g->d_h + g->d_w != head_dim) return VA3D_ERR_INVALID;
    if (!(g->theta > 0.0) || !std::isfinite(g->theta)) return VA3D_ERR_INVALID;
    const long long nv = static_cast<long long>(g->T) * g->H * g->W;
    if (nv + g->n_text != N) return VA3D_ERR_INVALID;
    return VA3D_OK;
}

int check_sizes(int B, int heads, int N, int head_dim) {
    if (B < 1 || heads < 1 || N < 1) return VA3D_ERR_INVALID;
    if (head_dim != kHeadDim) return VA3D_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * heads > 65535) return VA3D_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * heads * N * kHeadDim * 2 > (1ll << 40)) return VA3D_ERR_UNSUPPORTED;
    return VA3D_OK;
}

// Per-device facts every launch needs (architecture check, SM count, the
// dynamic shared-memory limit already granted to each kernel), looked up
// once per device under a mutex instead of on every call.
constexpr int kMaxDevices = 64;
enum KernelSlot {
    K_ATTN2, K_ATTN1, K_TEMP64R, K_TEMP64K,
    K_TTC0,   // temporal_tc_kernel<R, raw>: K_TTC0 + 2 * log2(R / 8) + (raw ? 0 : 1)
    NUM_KERNEL_SLOTS = K_TTC0 + 6
};

struct DeviceInfo {
    int state;                     // 0 unknown, 1 sm_100, 2 other architecture
    int sms;
    int smem_set[NUM_KERNEL_SLOTS];   // dynamic shared memory granted so far
};
DeviceInfo g_devices[kMaxDevices] = {};
std::mutex g_devices_mutex;

int current_device(int *dev) {
    if (cudaGetDevice(dev) != cudaSuccess) return VA3D_ERR_CUDA;
    if (*dev < 0 || *dev >= kMaxDevices) return VA3D_ERR_UNSUPPORTED;
    return VA3D_OK;
}

int check_device() {
    int dev = 0, rc;
    if ((rc = current_device(&dev)) != VA3D_OK) return rc;
    std::lock_guard<std::mutex> lock(g_devices_mutex);
    DeviceInfo &d = g_devices[dev];
    if (d.state == 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return VA3D_ERR_CUDA;
        d.sms = sms;
        d.state = (major == 10 && minor == 0) ? 1 : 2;
    }
    return d.state == 1 ? VA3D_OK : VA3D_ERR_DEVICE;
}

// SM count of the current device (after check_device() succeeded on it).
int device_sms(int *sms) {
    int dev = 0, rc;
    if ((rc = check_device()) != VA3D_OK) return rc;
    if ((rc = current_device(&dev)) != VA3D_OK) return rc;
    std::lock_guard<std::mutex> lock(g_devices_mutex);
    *sms = g_devices[dev].sms;
    return VA3D_OK;
}

// Grant `kernel` (slot `slot`) at least `bytes` of dynamic shared memory on
// the current device; the attribute is set only when the need grows.
int grant_smem(const void *kernel, int slot, int bytes) {
    int dev = 0, rc;
    if ((rc = current_device(&dev)) != VA3D_OK) return rc;
    std::lock_guard<std::mutex> lock(g_devices_mutex);
    int &set = g_devices[dev].smem_set[slot];
    if (bytes <= set) return VA3D_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return VA3D_ERR_CUDA;
    set = bytes;
    return VA3D_OK;
}

long long table_entries(const va3d_grid_t *g) {
    return static_cast<long long>(g->T) * (g->d_t / 2) + static_cast<long long>(g->H) * (g->d_h / 2) +
           static_cast<long long>(g->W) * (g->d_w / 2);
}

size_t table_bytes(const va3d_grid_t *g) { return round_up(8 * table_entries(g), 256); }

size_t tensor_bytes(int B, int heads, int N) {
    return static_cast<size_t>(B) * heads * N * kHeadDim * 2;
}

// Scratch for tiles of the last wave split over two key halves: per tile two
// normalised fp32 partial outputs of 256 rows, their (max, sum) and a counter.
// At most kMaxSplit tiles are split (half of the SMs of a GPU with up to 256).
constexpr int kMaxSplit = 128;
// Segments of at most this many 128-key tiles (e.g. text cross-attention over
// up to 512 text tokens) run one query tile per CTA, two CTAs per SM: there
// the per-CTA prologue and epilogue weigh most and overlapping them across
// CTAs pays (+10 % at 4 key tiles).  Longer segments keep two tiles per CTA
// (one CTA per SM is 10-15 % faster from 29 key tiles on), and so do windows,
// whose gathered K/V rows would be fetched twice as often.
constexpr int kOneTileMaxKeyTiles = 4;
constexpr size_t kSplitOBytes = 2 * 256 * 128 * 4;
constexpr size_t kSplitMLBytes = 2 * 256 * 8;

long long attn_tiles(int BH, int N) {
    return static_cast<long long>(BH) * ((N + 255) / 256);
}

size_t split_bytes_for(long long tiles) {
    const long long n = std::min<long long>(kMaxSplit, tiles);
    return round_up(static_cast<size_t>(n) * (kSplitOBytes + kSplitMLBytes + 4), 256);
}

RopeParams make_rope_params(const va3d_grid_t *g) {
    RopeParams rp;
    std::memset(&rp, 0, sizeof rp);
    rp.T = g->T;
    rp.H = g->H;
    rp.W = g->W;
    rp.HW = g->H * g->W;
    rp.n_video = g->T * g->H * g->W;
    rp.half_t = g->d_t / 2;
    rp.half_h = g->d_h / 2;
    rp.half_w = g->d_w / 2;
    rp.pe_t = rp.half_t;
    rp.pe_h = rp.half_t + rp.half_h;
    rp.tab_h = g->T * rp.half_t;
    rp.tab_w = rp.tab_h + g->H * rp.half_h;
    rp.tab_entries = rp.tab_w + g->W * rp.half_w;
    // inverse frequency of every pair: theta^(-2j/d) for index j in its axis range
    const int dims[3] = {g->d_t, g->d_h, g->d_w};
    int p = 0;
    for (int ax = 0; ax < 3; ++ax)
        for (int j = 0; j < dims[ax] / 2; ++j, ++p)
            rp.inv_freq[p] = static_cast<float>(std::pow(g->theta, -2.0 * j / dims[ax]));
    return rp;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// [BH, N, 128] bf16 viewed as a 3D tensor (dim, row, bh); boxes of
// 64 columns x box_rows rows with the 128-byte swizzle; rows past N read as zero.
// Encoding is a pure host computation of (base, N, BH, box_rows), so the
// last maps encoded are kept (a small direct-mapped cache under a mutex).
int encode_map(CUtensorMap *map, const void *base, int N, int BH, int box_rows);

// The temporal pass's view of [BH, T*HW, 128] bf16: a 4D tensor (dim, frame,
// position, bh) whose frames are HW rows apart; boxes of 64 dims x R frames x
// P positions (frames past T and positions past HW read as zero), 128-byte
// swizzle.
int encode_map_tp(CUtensorMap *map, const void *base, int T, int HW, int BH, int R, int P);

struct MapSlot {
    const void *base;
    int N, BH, box_rows;
    int T, HW, P;   // temporal-pass maps (box_rows = R); 0 for the 3D maps
    CUtensorMap map;
};
constexpr int kMapSlots = 64;
MapSlot g_map_slots[kMapSlots] = {};
std::mutex g_map_mutex;

// Cached encoding: (T, HW, P) = (0, 0, 0) selects the 3D map of
// encode_map, otherwise the temporal-pass map of encode_map_tp (N = T * HW).
int make_map_any(CUtensorMap *map, const void *base, int N, int BH, int box_rows, int T, int HW, int P) {
    const uintptr_t key = reinterpret_cast<uintptr_t>(base) ^ (static_cast<uintptr_t>(N) * 0x9E3779B1u) ^
                          (static_cast<uintptr_t>(BH) << 7) ^ static_cast<uintptr_t>(box_rows) ^
                          (static_cast<uintptr_t>(P) << 13);
    MapSlot &slot = g_map_slots[(key ^ (key >> 17) ^ (key >> 31)) % kMapSlots];
    std::lock_guard<std::mutex> lock(g_map_mutex);
    if (slot.base == base && slot.N == N && slot.BH == BH && slot.box_rows == box_rows && slot.T == T &&
        slot.HW == HW && slot.P == P && base != nullptr) {
        *map = slot.map;
        return VA3D_OK;
    }
    const int rc = P == 0 ? encode_map(map, base, N, BH, box_rows)
                          : encode_map_tp(map, base, T, HW, BH, box_rows, P);
    if (rc != VA3D_OK) return rc;
    slot.base = base;
    slot.N = N;
    slot.BH = BH;
    slot.box_rows = box_rows;
    slot.T = T;
    slot.HW = HW;
    slot.P = P;
    slot.map = *map;
    return VA3D_OK;
}

int make_map(CUtensorMap *map, const void *base, int N, int BH, int box_rows) {
    return make_map_any(map, base, N, BH, box_rows, 0, 0, 0);
}

int encode_map_tp(CUtensorMap *map, const void *base, int T, int HW, int BH, int R, int P) {
    auto fn = encode_fn();
    if (fn == nullptr) return VA3D_ERR_CUDA;
    const cuuint64_t row = static_cast<cuuint64_t>(kHeadDim) * 2;   // bytes per token row
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(T),
                          static_cast<cuuint64_t>(HW), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[3] = {row * static_cast<cuuint64_t>(HW), row,
                             row * static_cast<cuuint64_t>(T) * static_cast<cuuint64_t>(HW)};
    cuuint32_t box[4] = {64, static_cast<cuuint32_t>(R), static_cast<cuuint32_t>(P), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? VA3D_OK : VA3D_ERR_CUDA;
}

int encode_map(CUtensorMap *map, const void *base, int N, int BH, int box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return VA3D_ERR_CUDA;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * 2,
                             static_cast<cuuint64_t>(N) * kHeadDim * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? VA3D_OK : VA3D_ERR_CUDA;
}

// Shapes of a Ulysses exchange: the attention limits on whole sequences
// (B, heads/world, N) and on the local slices (B, heads, N/world).
int check_ulysses(int B, int heads, int N, int head_dim, int world) {
    if (world < 1 || world > cp::kMaxWorld) return VA3D_ERR_UNSUPPORTED;
    int rc;
    if ((rc = check_sizes(B, heads, N, head_dim)) != VA3D_OK) return rc;
    if (heads % world != 0 || N % world != 0) return VA3D_ERR_UNSUPPORTED;
    return VA3D_OK;
}

int check_ring(int B, int heads, int N, int head_dim, int world) {
    if (world < 1 || world > cp::kMaxWorld) return VA3D_ERR_UNSUPPORTED;
    int rc;
    if ((rc = check_sizes(B, heads, N, head_dim)) != VA3D_OK) return rc;
    if (N % world != 0) return VA3D_ERR_UNSUPPORTED;
    return VA3D_OK;
}

bool aligned256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

int check_regions(void *const *regions, int world, int rank) {
    if (regions == nullptr || rank < 0 || rank >= world) return VA3D_ERR_INVALID;
    for (int j = 0; j < world; ++j) {
        if (regions[j] == nullptr) return VA3D_ERR_INVALID;
        if ((reinterpret_cast<uintptr_t>(regions[j]) & 255u) != 0) return VA3D_ERR_ALIGNMENT;
    }
    return VA3D_OK;
}

int launch_status() {
    return cudaGetLastError() == cudaSuccess ? VA3D_OK : VA3D_ERR_CUDA;
}

int launch_table(float2 *tab, int *zero, int n_zero, const RopeParams &rp, cudaStream_t st) {
    const int work = std::max(rp.tab_entries, n_zero);
    if (work == 0) return VA3D_OK;
    const int threads = 256;
    const int blocks = (work + threads - 1) / threads;
    rope_table_kernel<<<blocks, threads, 0, st>>>(tab, zero, n_zero, rp);
    return launch_status();
}

// zero, n_zero: split-tail counters of the attention launch that follows,
// cleared by the same launch (optional).
int launch_rope(const void *x, void *y, int BH, int N, const RopeParams &rp, cudaStream_t st,
                int *zero = nullptr, int n_zero = 0) {
    const long long threads = static_cast<long long>(N) * 16;
    const long long blocks = (threads + kRopeThreads - 1) / kRopeThreads;
    rope_apply_kernel<<<static_cast<unsigned>(blocks), kRopeThreads, 0, st>>>(
        static_cast<const uint4 *>(x), static_cast<uint4 *>(y), N, BH, rp, zero, n_zero);
    return launch_status();
}

// Attention over segments of seg_len tokens (n_seg * seg_len == n_video or N).
// Split scratch region: kMaxSplit partial outputs, then (max, sum) pairs,
// then counters (cleared by the table kernel before every launch).
struct SplitScratch {
    float *part_o;
    float2 *part_ml;
    int *count;
    int capacity;   // tiles that fit
};

SplitScratch split_scratch(void *base, size_t bytes) {
    SplitScratch sc;
    const size_t per = kSplitOBytes + kSplitMLBytes + 4;
    sc.capacity = base == nullptr ? 0 : static_cast<int>(std::min<size_t>(kMaxSplit, bytes / per));
    uint8_t *p = static_cast<uint8_t *>(base);
    sc.part_o = reinterpret_cast<float *>(p);
    sc.part_ml = reinterpret_cast<float2 *>(p + sc.capacity * kSplitOBytes);
    sc.count = reinterpret_cast<int *>(p + sc.capacity * (kSplitOBytes + kSplitMLBytes));
    return sc;
}

// Q is [BH, N, 128] in n_seg segments of seg_len rows; K and V are
// [BH, Nkv, 128] in n_seg segments of kv_len rows; segment s of the queries
// attends to segment s of the keys.
// win (optional): local 3D window size; segments are then the windows, their
// rows gathered token by token (seg_len == kv_len == window volume).
// merge (optional): the ring form's log-sum-exp merge into an accumulator,
// done in the kernel's epilogue (no tile is split then).
struct RingMerge {
    int merge;            // 1: first block, 2: merge with lse_in
    float *acc;
    const float *lse_in;
    float *lse_out;
};

int launch_attn(const void *q, const void *k_rot, const void *v, void *o, float *lse, int BH, int N,
                int Nkv, int seg_len, int kv_len, int n_seg, bool rope_q, const RopeParams &rp,
                const float2 *tab, float scale, const SplitScratch &sc, cudaStream_t st,
                const int *win = nullptr, const RingMerge *merge = nullptr) {
    CUtensorMap mq, mk, mv;
    int rc;
    // windows whose width is a multiple of 8 dividing 128 load their rows as
    // TMA boxes of one run (win_w consecutive tokens) each
    const bool win_runs = win != nullptr && win[2] % 8 == 0 && fa::BM % win[2] == 0;
    const int qrows = win_runs ? win[2] : fa::BM, krows = win_runs ? win[2] : fa::BN;
    if ((rc = make_map(&mq, q, N, BH, qrows)) != VA3D_OK) return rc;
    if ((rc = make_map(&mk, k_rot, Nkv, BH, krows)) != VA3D_OK) return rc;
    if ((rc = make_map(&mv, v, Nkv, BH, krows)) != VA3D_OK) return rc;
    fa::AttnArgs a;
    std::memset(&a, 0, sizeof a);
    a.N = N;
    a.seg_len = seg_len;
    a.kv_len = kv_len;
    // two query tiles per CTA for long key sequences; one (two CTAs per SM)
    // when a unit's key loop is short and its prologue and epilogue weigh
    const int n_kv_tiles = (kv_len + fa::BN - 1) / fa::BN;
    const int nq = win == nullptr && n_kv_tiles <= kOneTileMaxKeyTiles ? 1 : 2;
    a.q_blocks = (seg_len + nq * fa::BM - 1) / (nq * fa::BM);
    a.scale_log2 = static_cast<float>(scale * kLog2e);
    a.rope_q = rope_q ? 1 : 0;
    a.o = static_cast<__nv_bfloat16 *>(o);
    a.lse = lse;
    a.rp = rp;
    if (win != nullptr) {
        a.win = win_runs ? 2 : 1;
        a.win_t = win[0];
        a.win_h = win[1];
        a.win_w = win[2];
        a.nwin_h = rp.H / win[1];
        a.nwin_w = rp.W / win[2];
        a.gq = static_cast<const __nv_bfloat16 *>(q);
        a.gk = static_cast<const __nv_bfloat16 *>(k_rot);
        a.gv = static_cast<const __nv_bfloat16 *>(v);
    }
    a.n_seg = n_seg;
    if (merge != nullptr) {
        a.merge = merge->merge;
        a.acc = merge->acc;
        a.lse_in = merge->lse_in;
        a.lse_out = merge->lse_out;
    }
    // O by TMA store: segments that tile the rows (boxes clipped at each
    // segment's end), or window runs; the ring merge writes rows itself
    CUtensorMap mo;
    std::memset(&mo, 0, sizeof mo);
    if (merge == nullptr && o != nullptr) {
        if (win_runs) {
            if ((rc = make_map(&mo, o, N, BH, win[2])) != VA3D_OK) return rc;
            a.o_tma = 2;
        } else if (win == nullptr && static_cast<long long>(seg_len) * n_seg == N) {
            if ((rc = make_map(&mo, o, seg_len, n_seg * BH, fa::BM)) != VA3D_OK) return rc;
            a.o_tma = 1;
        }
    }
    // One CTA per SM.  If the last wave of tiles would fill at most half of the
    // SMs and every tile has at least two 128-key steps, each of its tiles is
    // covered by two units over half of the keys instead.
    int sms = 0;
    if ((rc = device_sms(&sms)) != VA3D_OK) return rc;
    const long long tiles = static_cast<long long>(BH) * n_seg * a.q_blocks;
    const long long resident = static_cast<long long>(sms) * (nq == 2 ? fa::KCfg<2>::kMinBlocks
                                                                      : fa::KCfg<1>::kMinBlocks);
    const long long tail = resident > 0 ? tiles % resident : 0;
    const int n_kv = (kv_len + fa::BN - 1) / fa::BN;
    long long split = 0;
    if (merge == nullptr && tail > 0 && 2 * tail <= resident && tail <= sc.capacity && n_kv >= 2)
        split = tail;
    a.n_whole = static_cast<int>(tiles - split);
    a.part_o = sc.part_o;
    a.part_ml = sc.part_ml;
    a.part_count = sc.count;
    const long long units = tiles + split;
    if (units > 0x7fffffffll) return VA3D_ERR_UNSUPPORTED;
    if (nq == 2) {
        using C = fa::KCfg<2>;
        if ((rc = grant_smem(reinterpret_cast<const void *>(fa::attn_fwd_kernel<2>), K_ATTN2,
                             C::kSmemBytes)) != VA3D_OK)
            return rc;
        fa::attn_fwd_kernel<2><<<static_cast<unsigned>(units), C::kThreads, C::kSmemBytes, st>>>(
            mq, mk, mv, mo, a);
    } else {
        using C = fa::KCfg<1>;
        if ((rc = grant_smem(reinterpret_cast<const void *>(fa::attn_fwd_kernel<1>), K_ATTN1,
                             C::kSmemBytes)) != VA3D_OK)
            return rc;
        fa::attn_fwd_kernel<1><<<static_cast<unsigned>(units), C::kThreads, C::kSmemBytes, st>>>(
            mq, mk, mv, mo, a);
    }
    return launch_status();
}

template <int MAXT, bool kRawK>
int launch_temporal_t(const tp::TemporalArgs &a, cudaStream_t st) {
    int sms = 0, rc;
    if ((rc = device_sms(&sms)) != VA3D_OK) return rc;
    // Warps per block and blocks per SM from the shared-memory budget; the
    // grid is persistent (at most the resident blocks), each warp strides
    // over (batch*head, position) tasks.
    const int warp_bytes = tp::temporal_warp_bytes(a.T);
    const int table_bytes = tp::temporal_table_bytes(a.T, a.rp.half_t);
    const int budget = tp::Cfg<MAXT>::kSmemBudget - table_bytes;
    const int warps = std::max(1, std::min(tp::Cfg<MAXT>::kMaxWarps, budget / warp_bytes));
    const int smem = table_bytes + warps * warp_bytes;
    const int per_sm = std::max(1, std::min(4, (216 * 1024) / smem));
    static_assert(MAXT == 64, "T' <= 32 runs on the tensor-core pass");
    constexpr int slot = kRawK ? K_TEMP64R : K_TEMP64K;
    if ((rc = grant_smem(reinterpret_cast<const void *>(tp::temporal_kernel<MAXT, kRawK>), slot, smem)) !=
        VA3D_OK)
        return rc;
    const long long tasks = static_cast<long long>(a.BH) * a.HW;
    const long long need = (tasks + warps - 1) / warps;
    const long long blocks = std::min<long long>(need, static_cast<long long>(sms) * per_sm);
    tp::temporal_kernel<MAXT, kRawK><<<static_cast<unsigned>(blocks), warps * 32, smem, st>>>(a);
    return launch_status();
}

// Tensor-core temporal pass (T' <= 32): one persistent block per SM, each
// block's two groups taking alternate tiles of P positions.
template <int R, bool kRawK>
int launch_temporal_tc_t(const tp::TemporalArgs &a, cudaStream_t st) {
    constexpr int P = tpc::Geo<R>::P;
    int sms = 0, rc;
    if ((rc = device_sms(&sms)) != VA3D_OK) return rc;
    CUtensorMap mq, mk, mv, mo;
    if ((rc = make_map_any(&mq, a.q, a.N, a.BH, R, a.T, a.HW, P)) != VA3D_OK) return rc;
    if ((rc = make_map_any(&mk, a.k, a.N, a.BH, R, a.T, a.HW, P)) != VA3D_OK) return rc;
    if ((rc = make_map_any(&mv, a.v, a.N, a.BH, R, a.T, a.HW, P)) != VA3D_OK) return rc;
    if ((rc = make_map_any(&mo, a.o, a.N, a.BH, R, a.T, a.HW, P)) != VA3D_OK) return rc;
    const int smem = tpc::smem_bytes(a.T, a.rp.pe_t, kRawK);
    constexpr int slot = K_TTC0 + 2 * (R == 8 ? 0 : (R == 16 ? 1 : 2)) + (kRawK ? 0 : 1);
    if ((rc = grant_smem(reinterpret_cast<const void *>(tpc::temporal_tc_kernel<R, kRawK>), slot, smem)) !=
        VA3D_OK)
        return rc;
    const long long tiles = static_cast<long long>(a.BH) * ((a.HW + P - 1) / P);
    if (tiles >= (1ll << 30)) return VA3D_ERR_UNSUPPORTED;   // tile indices are 32-bit
    const long long blocks = std::min<long long>(tiles, sms);
    tpc::temporal_tc_kernel<R, kRawK><<<static_cast<unsigned>(blocks), tpc::kThreads, smem, st>>>(mq, mk, mv, mo, a);
    return launch_status();
}

template <bool kRawK>
int launch_temporal_tc(const tp::TemporalArgs &a, cudaStream_t st) {
    switch (tpc::rows_per_position(a.T)) {
    case 8: return launch_temporal_tc_t<8, kRawK>(a, st);
    case 16: return launch_temporal_tc_t<16, kRawK>(a, st);
    default: return launch_temporal_tc_t<32, kRawK>(a, st);
    }
}

// k is the raw key tensor (rotated here) unless k_rotated.
int launch_temporal(const void *q, const void *k, bool k_rotated, const void *v, void *o, int BH,
                    int N, const RopeParams &rp, const float2 *tab, float scale, cudaStream_t st) {
    tp::TemporalArgs a;
    std::memset(&a, 0, sizeof a);
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.k = static_cast<const __nv_bfloat16 *>(k);
    a.v = static_cast<const __nv_bfloat16 *>(v);
    a.o = static_cast<__nv_bfloat16 *>(o);
    a.N = N;
    a.T = rp.T;
    a.HW = rp.HW;
    a.BH = BH;
    a.scale_log2 = static_cast<float>(scale * kLog2e);
    a.rope_k = k_rotated ? 0 : 1;
    a.rope_tab = tab;
    a.rp = rp;
    if (rp.T <= 32) return k_rotated ? launch_temporal_tc<false>(a, st) : launch_temporal_tc<true>(a, st);
    return k_rotated ? launch_temporal_t<64, false>(a, st) : launch_temporal_t<64, true>(a, st);
}

// Shared front half of the two attention entry points: checks, workspace
// split, angle table and (unless the keys come rotated) the key pre-pass.
struct Prepared {
    RopeParams rp;
    const float2 *tab;
    const void *k_rot;
    float scale;
    SplitScratch split;
};

// Workspace bytes a call cannot do without: the angle table and, unless the
// keys come rotated, the rotated keys.  The split scratch behind them is
// optional (split_scratch() sizes it from what is left).
size_t required_workspace_bytes(int B, int heads, int N, const va3d_grid_t *grid, unsigned flags) {
    return table_bytes(grid) + ((flags & VA3D_K_ROTATED) ? 0 : tensor_bytes(B, heads, N));
}

// split_optional: accept a workspace that holds only the required part (the
// built-in scratch of the no-allocation entry point); the public entry
// points ask for the full va3d_workspace_bytes().
// need_table: build the angle table (only the temporal pass reads it; the
// attention kernel forms its angles with the hardware sine and cosine).
// The split-tail counters are cleared by whichever of the table kernel or the
// key pre-pass runs, else by a clearing launch of the table kernel alone.
int prepare(const void *q, const void *k, const void *v, int B, int heads, int N, int head_dim,
            const va3d_grid_t *grid, float softmax_scale, unsigned flags, void *workspace,
            size_t workspace_bytes, bool need_k_rot, bool need_table, cudaStream_t st, Prepared *out,
            bool split_optional = false) {
    int rc;
    if ((rc = check_sizes(B, heads, N, head_dim)) != VA3D_OK) return rc;
    if ((rc = check_grid(grid, N, head_dim)) != VA3D_OK) return rc;
    if (q == nullptr || k == nullptr || v == nullptr) return VA3D_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return VA3D_ERR_ALIGNMENT;
    if (flags & ~static_cast<unsigned>(VA3D_K_ROTATED)) return VA3D_ERR_INVALID;
    const size_t need = split_optional ? required_workspace_bytes(B, heads, N, grid, flags)
                                       : va3d_workspace_bytes(B, heads, N, head_dim, grid, flags);
    if (workspace == nullptr || workspace_bytes < need) return VA3D_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return VA3D_ERR_ALIGNMENT;
    if ((rc = check_device()) != VA3D_OK) return rc;

    out->rp = make_rope_params(grid);
    out->tab = static_cast<const float2 *>(workspace);
    out->scale = softmax_scale > 0.f ? softmax_scale : static_cast<float>(1.0 / std::sqrt(double(head_dim)));
    // workspace: [angle table | rotated keys (unless given) | split scratch]
    size_t used = required_workspace_bytes(B, heads, N, grid, flags);
    out->split = split_scratch(used < workspace_bytes ? static_cast<uint8_t *>(workspace) + used : nullptr,
                               used < workspace_bytes ? workspace_bytes - used : 0);
    const bool prepass = !(flags & VA3D_K_ROTATED) && need_k_rot;
    if (need_table || (!prepass && out->split.capacity > 0)) {
        RopeParams tab_rp = out->rp;
        if (!need_table) tab_rp.tab_entries = 0;   // counters only
        if ((rc = launch_table(static_cast<float2 *>(workspace), prepass ? nullptr : out->split.count,
                               prepass ? 0 : out->split.capacity, tab_rp, st)) != VA3D_OK)
            return rc;
    }
    if (flags & VA3D_K_ROTATED) {
        out->k_rot = k;
    } else if (!need_k_rot) {
        out->k_rot = nullptr;
    } else {
        void *kr = static_cast<uint8_t *>(workspace) + table_bytes(grid);
        if ((rc = launch_rope(k, kr, B * heads, N, out->rp, st, out->split.count, out->split.capacity)) !=
            VA3D_OK)
            return rc;
        out->k_rot = kr;
    }
    return VA3D_OK;
}

}  // namespace

extern "C" {

const char *va3d_status_string(int status) {
    switch (status) {
    case VA3D_OK: return "success";
    case VA3D_ERR_INVALID: return "invalid argument (null pointer, size or grid)";
    case VA3D_ERR_UNSUPPORTED: return "unsupported size (head_dim must be 128; see limits)";
    case VA3D_ERR_ALIGNMENT: return "pointer not 16-byte aligned (workspace: 256-byte)";
    case VA3D_ERR_WORKSPACE: return "workspace missing or too small";
    case VA3D_ERR_CUDA: return "CUDA runtime or driver call failed";
    case VA3D_ERR_DEVICE: return "current device is not compute capability 10.0 (B200)";
    case VA3D_ERR_SCRATCH_LIMIT:
        return "problem needs more scratch than the 64 MiB built into attn3d_full_fwd_noalloc";
    default: return "unknown status";
    }
}

int va3d_version(void) { return 100; }

int va3d_grid_from_video(int frames, int height, int width, int d_t, int d_h, int d_w, int n_text,
                         va3d_grid_t *out) {
    if (out == nullptr || frames < 1 || height < 16 || width < 16 || n_text < 0) return VA3D_ERR_INVALID;
    if ((frames - 1) % 4 != 0 || height % 16 != 0 || width % 16 != 0) return VA3D_ERR_INVALID;
    va3d_grid_t g;
    g.T = 1 + (frames - 1) / 4;
    g.H = height / 16;
    g.W = width / 16;
    g.n_text = n_text;
    g.d_t = d_t;
    g.d_h = d_h;
    g.d_w = d_w;
    g.theta = 10000.0;
    *out = g;
    return VA3D_OK;
}

size_t va3d_workspace_bytes(int B, int heads, int N, int head_dim, const va3d_grid_t *grid,
                            unsigned flags) {
    if (check_sizes(B, heads, N, head_dim) != VA3D_OK) return 0;
    if (check_grid(grid, N, head_dim) != VA3D_OK) return 0;
    size_t bytes = table_bytes(grid);
    if (!(flags & VA3D_K_ROTATED)) bytes += tensor_bytes(B, heads, N);
    bytes += split_bytes_for(attn_tiles(B * heads, N));
    return bytes;
}

int rope3d_apply(const va3d_bf16 *x, va3d_bf16 *y, int B, int heads, int N, int head_dim,
                 const va3d_grid_t *grid, void *stream) {
    TraceRange trace("va3d.rope3d_apply");
    int rc;
    if ((rc = check_sizes(B, heads, N, head_dim)) != VA3D_OK) return rc;
    if ((rc = check_grid(grid, N, head_dim)) != VA3D_OK) return rc;
    if (x == nullptr || y == nullptr) return VA3D_ERR_INVALID;
    if (!aligned16(x) || !aligned16(y)) return VA3D_ERR_ALIGNMENT;
    if ((rc = check_device()) != VA3D_OK) return rc;
    return launch_rope(x, y, B * heads, N, make_rope_params(grid), static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

int full_fwd(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v, va3d_bf16 *o, float *lse,
             int B, int heads, int N, int head_dim, const va3d_grid_t *grid, float softmax_scale,
             unsigned flags, void *workspace, size_t workspace_bytes, void *stream,
             bool split_optional) {
    if (o == nullptr) return VA3D_ERR_INVALID;
    if (!aligned16(o) || (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return VA3D_ERR_ALIGNMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Prepared p;
    int rc = prepare(q, k, v, B, heads, N, head_dim, grid, softmax_scale, flags, workspace,
                     workspace_bytes, true, false, st, &p, split_optional);
    if (rc != VA3D_OK) return rc;
    return launch_attn(q, p.k_rot, v, o, lse, B * heads, N, N, N, N, 1, true, p.rp, p.tab, p.scale,
                       p.split, st);
}

}  // namespace

extern "C" {

int attn3d_full_fwd(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v, va3d_bf16 *o,
                    float *lse, int B, int heads, int N, int head_dim, const va3d_grid_t *grid,
                    float softmax_scale, unsigned flags, void *workspace, size_t workspace_bytes,
                    void *stream) {
    TraceRange trace("va3d.attn3d_full_fwd");
    return full_fwd(q, k, v, o, lse, B, heads, N, head_dim, grid, softmax_scale, flags, workspace,
                    workspace_bytes, stream, false);
}

int attn_factorized_fwd(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v,
                        va3d_bf16 *o_spatial, va3d_bf16 *o_temporal, int B, int heads, int N,
                        int head_dim, const va3d_grid_t *grid, float softmax_scale, unsigned flags,
                        void *workspace, size_t workspace_bytes, void *stream) {
    TraceRange trace("va3d.attn_factorized_fwd");
    if (o_spatial == nullptr && o_temporal == nullptr) return VA3D_ERR_INVALID;
    if ((o_spatial && !aligned16(o_spatial)) || (o_temporal && !aligned16(o_temporal)))
        return VA3D_ERR_ALIGNMENT;
    if (grid == nullptr) return VA3D_ERR_INVALID;
    if (grid->n_text != 0) return VA3D_ERR_INVALID;
    if (o_temporal != nullptr && grid->T > 64) return VA3D_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Prepared p;
    int rc = prepare(q, k, v, B, heads, N, head_dim, grid, softmax_scale, flags, workspace,
                     workspace_bytes, o_spatial != nullptr, o_temporal != nullptr, st, &p);
    if (rc != VA3D_OK) return rc;
    if (o_spatial != nullptr) {
        rc = launch_attn(q, p.k_rot, v, o_spatial, nullptr, B * heads, N, N, p.rp.HW, p.rp.HW,
                         p.rp.T, true, p.rp, p.tab, p.scale, p.split, st);
        if (rc != VA3D_OK) return rc;
    }
    if (o_temporal != nullptr)
        rc = launch_temporal(q, k, (flags & VA3D_K_ROTATED) != 0, v, o_temporal, B * heads, N, p.rp,
                             p.tab, p.scale, st);
    return rc;
}

size_t va3d_cross_workspace_bytes(int B, int heads, int Nq, int Nkv, int head_dim) {
    if (check_sizes(B, heads, Nq, head_dim) != VA3D_OK) return 0;
    if (check_sizes(B, heads, Nkv, head_dim) != VA3D_OK) return 0;
    return split_bytes_for(attn_tiles(B * heads, Nq));
}

int attn_cross_fwd(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v, va3d_bf16 *o,
                   float *lse, int B, int heads, int Nq, int Nkv, int head_dim, float softmax_scale,
                   void *workspace, size_t workspace_bytes, void *stream) {
    TraceRange trace("va3d.attn_cross_fwd");
    int rc;
    if ((rc = check_sizes(B, heads, Nq, head_dim)) != VA3D_OK) return rc;
    if ((rc = check_sizes(B, heads, Nkv, head_dim)) != VA3D_OK) return rc;
    if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return VA3D_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
        (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return VA3D_ERR_ALIGNMENT;
    if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return VA3D_ERR_ALIGNMENT;
    if ((rc = check_device()) != VA3D_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const float scale =
        softmax_scale > 0.f ? softmax_scale : static_cast<float>(1.0 / std::sqrt(double(head_dim)));
    // The workspace only holds the scratch for splitting the last wave's
    // tiles; without one (or with too little) those tiles run whole.
    SplitScratch sc = split_scratch(workspace, workspace != nullptr ? workspace_bytes : 0);
    RopeParams none;
    std::memset(&none, 0, sizeof none);
    if ((rc = launch_table(nullptr, sc.count, sc.capacity, none, st)) != VA3D_OK) return rc;
    return launch_attn(q, k, v, o, lse, B * heads, Nq, Nkv, Nq, Nkv, 1, false, none, nullptr, scale,
                       sc, st);
}

int attn_window_fwd(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v, va3d_bf16 *o,
                    float *lse, int B, int heads, int N, int head_dim, const va3d_grid_t *grid,
                    int win_t, int win_h, int win_w, float softmax_scale, unsigned flags,
                    void *workspace, size_t workspace_bytes, void *stream) {
    TraceRange trace("va3d.attn_window_fwd");
    if (o == nullptr || grid == nullptr) return VA3D_ERR_INVALID;
    if (!aligned16(o) || (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return VA3D_ERR_ALIGNMENT;
    if (grid->n_text != 0 || win_t < 1 || win_h < 1 || win_w < 1) return VA3D_ERR_INVALID;
    if (grid->T % win_t != 0 || grid->H % win_h != 0 || grid->W % win_w != 0) return VA3D_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Prepared p;
    int rc = prepare(q, k, v, B, heads, N, head_dim, grid, softmax_scale, flags, workspace,
                     workspace_bytes, true, false, st, &p);
    if (rc != VA3D_OK) return rc;
    const int win[3] = {win_t, win_h, win_w};
    const int vol = win_t * win_h * win_w;
    return launch_attn(q, p.k_rot, v, o, lse, B * heads, N, N, vol, vol, N / vol, true, p.rp, p.tab,
                       p.scale, p.split, st, win);
}

int va3d_watchdog_selftest(void *stream) {
    int rc;
    if ((rc = check_device()) != VA3D_OK) return rc;
    watchdog_probe_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>();
    return launch_status();
}

int va3d_device_error(int reset) {
    if (cudaDeviceSynchronize() != cudaSuccess) return VA3D_ERR_CUDA;
    int value = 0;
    if (cudaMemcpyFromSymbol(&value, va3d::g_device_error, sizeof value) != cudaSuccess)
        return VA3D_ERR_CUDA;
    if (reset) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(va3d::g_device_error, &zero, sizeof zero) != cudaSuccess)
            return VA3D_ERR_CUDA;
    }
    return value;
}


size_t va3d_ulysses_region_bytes(int B, int heads, int N, int head_dim, int world) {
    if (check_ulysses(B, heads, N, head_dim, world) != VA3D_OK) return 0;
    return cp::region_layout(B, heads, N, world).bytes;
}

int va3d_ulysses_offsets(int B, int heads, int N, int head_dim, int world, size_t *off_q,
                         size_t *off_k, size_t *off_v, size_t *off_o) {
    int rc;
    if ((rc = check_ulysses(B, heads, N, head_dim, world)) != VA3D_OK) return rc;
    if (off_q == nullptr || off_k == nullptr || off_v == nullptr || off_o == nullptr)
        return VA3D_ERR_INVALID;
    const cp::Layout l = cp::region_layout(B, heads, N, world);
    *off_q = l.q;
    *off_k = l.k;
    *off_v = l.v;
    *off_o = l.o;
    return VA3D_OK;
}

int va3d_region_alloc(size_t bytes, void **ptr) {
    if (bytes == 0 || ptr == nullptr) return VA3D_ERR_INVALID;
    *ptr = nullptr;
    void *p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) return VA3D_ERR_CUDA;
    if (cudaMemset(p, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        cudaFree(p);
        return VA3D_ERR_CUDA;
    }
    *ptr = p;
    return VA3D_OK;
}

int va3d_region_free(void *ptr) {
    if (ptr == nullptr) return VA3D_ERR_INVALID;
    return cudaFree(ptr) == cudaSuccess ? VA3D_OK : VA3D_ERR_CUDA;
}

int va3d_ipc_export(const void *region, unsigned char *handle) {
    static_assert(sizeof(cudaIpcMemHandle_t) == VA3D_IPC_HANDLE_BYTES, "IPC handle size");
    if (region == nullptr || handle == nullptr) return VA3D_ERR_INVALID;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, const_cast<void *>(region)) != cudaSuccess) return VA3D_ERR_CUDA;
    std::memcpy(handle, &h, sizeof h);
    return VA3D_OK;
}

int va3d_ipc_open(const unsigned char *handle, void **ptr) {
    if (handle == nullptr || ptr == nullptr) return VA3D_ERR_INVALID;
    *ptr = nullptr;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof h);
    void *p = nullptr;
    if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return VA3D_ERR_CUDA;
    *ptr = p;
    return VA3D_OK;
}

int va3d_ipc_close(void *ptr) {
    if (ptr == nullptr) return VA3D_ERR_INVALID;
    return cudaIpcCloseMemHandle(ptr) == cudaSuccess ? VA3D_OK : VA3D_ERR_CUDA;
}

int va3d_ulysses_scatter(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v,
                         void *const *regions, int world, int rank, int B, int heads, int N,
                         int head_dim, const va3d_grid_t *grid, unsigned flags, void *stream) {
    TraceRange trace("va3d.va3d_ulysses_scatter");
    int rc;
    if ((rc = check_ulysses(B, heads, N, head_dim, world)) != VA3D_OK) return rc;
    if ((rc = check_grid(grid, N, head_dim)) != VA3D_OK) return rc;
    if ((rc = check_regions(regions, world, rank)) != VA3D_OK) return rc;
    if (q == nullptr || k == nullptr || v == nullptr) return VA3D_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return VA3D_ERR_ALIGNMENT;
    if (flags & ~static_cast<unsigned>(VA3D_K_ROTATED)) return VA3D_ERR_INVALID;
    if ((rc = check_device()) != VA3D_OK) return rc;
    const cp::Layout l = cp::region_layout(B, heads, N, world);
    cp::ScatterArgs a;
    std::memset(&a, 0, sizeof a);
    a.q = static_cast<const uint4 *>(static_cast<const void *>(q));
    a.k = static_cast<const uint4 *>(static_cast<const void *>(k));
    a.v = static_cast<const uint4 *>(static_cast<const void *>(v));
    for (int j = 0; j < world; ++j) a.region[j] = static_cast<uint8_t *>(regions[j]);
    a.off_q = l.q;
    a.off_k = l.k;
    a.off_v = l.v;
    a.world = world;
    a.rank = rank;
    a.B = B;
    a.heads = heads;
    a.hpw = heads / world;
    a.N = N;
    a.n_loc = N / world;
    a.rotate_k = (flags & VA3D_K_ROTATED) ? 0 : 1;
    const int blocks = cp::copy_blocks(a.n_loc);
    cp::ulysses_scatter_kernel<<<blocks, cp::kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        a, make_rope_params(grid));
    return launch_status();
}

int va3d_ulysses_gather(const va3d_bf16 *o_heads, void *const *regions, int world, int rank,
                        int B, int heads, int N, int head_dim, void *stream) {
    TraceRange trace("va3d.va3d_ulysses_gather");
    int rc;
    if ((rc = check_ulysses(B, heads, N, head_dim, world)) != VA3D_OK) return rc;
    if ((rc = check_regions(regions, world, rank)) != VA3D_OK) return rc;
    if (o_heads == nullptr) return VA3D_ERR_INVALID;
    if (!aligned16(o_heads)) return VA3D_ERR_ALIGNMENT;
    if ((rc = check_device()) != VA3D_OK) return rc;
    cp::GatherArgs a;
    std::memset(&a, 0, sizeof a);
    a.o = static_cast<const uint4 *>(static_cast<const void *>(o_heads));
    for (int j = 0; j < world; ++j) a.region[j] = static_cast<uint8_t *>(regions[j]);
    a.off_o = cp::region_layout(B, heads, N, world).o;
    a.world = world;
    a.rank = rank;
    a.B = B;
    a.heads = heads;
    a.hpw = heads / world;
    a.N = N;
    a.n_loc = N / world;
    const int blocks = cp::copy_blocks(N);
    cp::ulysses_gather_kernel<<<blocks, cp::kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return launch_status();
}

int va3d_ulysses_wait(const void *region, int phase, unsigned long long epoch, int world, int B,
                      int heads, int N, int head_dim, void *stream) {
    TraceRange trace("va3d.va3d_ulysses_wait");
    int rc;
    if ((rc = check_ulysses(B, heads, N, head_dim, world)) != VA3D_OK) return rc;
    if (region == nullptr || (phase != cp::kScatter && phase != cp::kGather) || epoch == 0)
        return VA3D_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(region) & 255u) != 0) return VA3D_ERR_ALIGNMENT;
    if ((rc = check_device()) != VA3D_OK) return rc;
    const int blocks = cp::copy_blocks(phase == cp::kScatter ? N / world : N);
    const unsigned long long expected = epoch * static_cast<unsigned long long>(world) * blocks;
    cp::ulysses_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const unsigned long long *>(region), phase, expected);
    return launch_status();
}

size_t va3d_ring_region_bytes(int B, int heads, int N, int head_dim, int world) {
    if (check_ring(B, heads, N, head_dim, world) != VA3D_OK) return 0;
    return ring::region_layout(B, heads, N, world).bytes;
}

int va3d_ring_offsets(int B, int heads, int N, int head_dim, int world, size_t *off_k0,
                      size_t *off_v0, size_t *off_k1, size_t *off_v1) {
    int rc;
    if ((rc = check_ring(B, heads, N, head_dim, world)) != VA3D_OK) return rc;
    if (off_k0 == nullptr || off_v0 == nullptr || off_k1 == nullptr || off_v1 == nullptr)
        return VA3D_ERR_INVALID;
    const ring::Layout l = ring::region_layout(B, heads, N, world);
    *off_k0 = l.k[0];
    *off_v0 = l.v[0];
    *off_k1 = l.k[1];
    *off_v1 = l.v[1];
    return VA3D_OK;
}

int va3d_ring_load(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v, va3d_bf16 *q_rot,
                   void *region, int world, int rank, int B, int heads, int N, int head_dim,
                   const va3d_grid_t *grid, unsigned flags, void *stream) {
    TraceRange trace("va3d.va3d_ring_load");
    int rc;
    if ((rc = check_ring(B, heads, N, head_dim, world)) != VA3D_OK) return rc;
    if ((rc = check_grid(grid, N, head_dim)) != VA3D_OK) return rc;
    if (q == nullptr || k == nullptr || v == nullptr || q_rot == nullptr || region == nullptr ||
        rank < 0 || rank >= world)
        return VA3D_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_rot) || !aligned256(region))
        return VA3D_ERR_ALIGNMENT;
    if (flags & ~static_cast<unsigned>(VA3D_K_ROTATED)) return VA3D_ERR_INVALID;
    if ((rc = check_device()) != VA3D_OK) return rc;
    const ring::Layout l = ring::region_layout(B, heads, N, world);
    uint8_t *base = static_cast<uint8_t *>(region);
    ring::LoadArgs a;
    a.q = static_cast<const uint4 *>(static_cast<const void *>(q));
    a.k = static_cast<const uint4 *>(static_cast<const void *>(k));
    a.v = static_cast<const uint4 *>(static_cast<const void *>(v));
    a.q_rot = static_cast<uint4 *>(static_cast<void *>(q_rot));
    a.k0 = reinterpret_cast<uint4 *>(base + l.k[0]);
    a.v0 = reinterpret_cast<uint4 *>(base + l.v[0]);
    a.rows = static_cast<long long>(B) * heads;
    a.n_loc = N / world;
    a.offset = rank * (N / world);
    a.rope_q = 1;
    a.rope_k = (flags & VA3D_K_ROTATED) ? 0 : 1;
    ring::ring_load_kernel<<<cp::copy_blocks(a.n_loc), cp::kCopyThreads, 0,
                             static_cast<cudaStream_t>(stream)>>>(a, make_rope_params(grid));
    return launch_status();
}

int va3d_ring_pass(const void *region, void *next_region, int buf, int world, int B, int heads,
                   int N, int head_dim, void *stream) {
    TraceRange trace("va3d.va3d_ring_pass");
    int rc;
    if ((rc = check_ring(B, heads, N, head_dim, world)) != VA3D_OK) return rc;
    if (region == nullptr || next_region == nullptr || (buf != 0 && buf != 1)) return VA3D_ERR_INVALID;
    if (!aligned256(region) || !aligned256(next_region)) return VA3D_ERR_ALIGNMENT;
    if ((rc = check_device()) != VA3D_OK) return rc;
    const ring::Layout l = ring::region_layout(B, heads, N, world);
    const uint8_t *src = static_cast<const uint8_t *>(region);
    uint8_t *dst = static_cast<uint8_t *>(next_region);
    const long long rows = static_cast<long long>(B) * heads * (N / world);
    ring::ring_pass_kernel<<<cp::copy_blocks(rows), cp::kCopyThreads, 0,
                             static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4 *>(src + l.k[buf]), reinterpret_cast<const uint4 *>(src + l.v[buf]),
        reinterpret_cast<uint4 *>(dst + l.k[1 - buf]), reinterpret_cast<uint4 *>(dst + l.v[1 - buf]),
        rows * 16, dst);
    return launch_status();
}

int va3d_ring_free(void *prev_region, void *stream) {
    TraceRange trace("va3d.va3d_ring_free");
    int rc;
    if (prev_region == nullptr) return VA3D_ERR_INVALID;
    if (!aligned256(prev_region)) return VA3D_ERR_ALIGNMENT;
    if ((rc = check_device()) != VA3D_OK) return rc;
    ring::ring_free_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint8_t *>(prev_region));
    return launch_status();
}

int va3d_ring_wait(const void *region, int counter, unsigned long long count, int world, int B,
                   int heads, int N, int head_dim, void *stream) {
    TraceRange trace("va3d.va3d_ring_wait");
    int rc;
    if ((rc = check_ring(B, heads, N, head_dim, world)) != VA3D_OK) return rc;
    if (region == nullptr || (counter != ring::kFull && counter != ring::kFree)) return VA3D_ERR_INVALID;
    if (!aligned256(region)) return VA3D_ERR_ALIGNMENT;
    if ((rc = check_device()) != VA3D_OK) return rc;
    const long long rows = static_cast<long long>(B) * heads * (N / world);
    const unsigned long long expected =
        counter == ring::kFull ? count * static_cast<unsigned long long>(cp::copy_blocks(rows)) : count;
    cp::ulysses_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const unsigned long long *>(region), counter, expected);
    return launch_status();
}

int va3d_ring_merge(const va3d_bf16 *o_blk, const float *lse_blk, float *acc, const float *lse_in,
                    float *lse_out, va3d_bf16 *out, int B, int heads, int n_rows, int first,
                    void *stream) {
    TraceRange trace("va3d.va3d_ring_merge");
    int rc;
    if ((rc = check_sizes(B, heads, n_rows, kHeadDim)) != VA3D_OK) return rc;
    if (o_blk == nullptr || lse_blk == nullptr || acc == nullptr || lse_out == nullptr ||
        (!first && lse_in == nullptr) || (!first && lse_in == lse_out))
        return VA3D_ERR_INVALID;
    if (!aligned16(o_blk) || !aligned16(acc) || (out != nullptr && !aligned16(out)) ||
        (reinterpret_cast<uintptr_t>(lse_blk) & 3u) || (reinterpret_cast<uintptr_t>(lse_out) & 3u) ||
        (lse_in != nullptr && (reinterpret_cast<uintptr_t>(lse_in) & 3u)))
        return VA3D_ERR_ALIGNMENT;
    if ((rc = check_device()) != VA3D_OK) return rc;
    const long long rows = static_cast<long long>(B) * heads * n_rows;
    ring::ring_merge_kernel<<<cp::copy_blocks(rows), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(static_cast<const void *>(o_blk)), lse_blk,
        reinterpret_cast<float4 *>(acc), lse_in, lse_out,
        out ? static_cast<uint4 *>(static_cast<void *>(out)) : nullptr, rows, first ? 1 : 0);
    return launch_status();
}

int va3d_ring_attend(const va3d_bf16 *q_rot, const va3d_bf16 *k, const va3d_bf16 *v, float *acc,
                     const float *lse_in, float *lse_out, va3d_bf16 *out, int B, int heads,
                     int n_rows, int n_keys, int head_dim, float softmax_scale, int first,
                     void *stream) {
    TraceRange trace("va3d.va3d_ring_attend");
    int rc;
    if ((rc = check_sizes(B, heads, n_rows, head_dim)) != VA3D_OK) return rc;
    if ((rc = check_sizes(B, heads, n_keys, head_dim)) != VA3D_OK) return rc;
    if (q_rot == nullptr || k == nullptr || v == nullptr || acc == nullptr || lse_out == nullptr ||
        (!first && lse_in == nullptr) || (!first && lse_in == lse_out))
        return VA3D_ERR_INVALID;
    if (!aligned16(q_rot) || !aligned16(k) || !aligned16(v) || !aligned16(acc) ||
        (out != nullptr && !aligned16(out)) || (reinterpret_cast<uintptr_t>(lse_out) & 3u) ||
        (lse_in != nullptr && (reinterpret_cast<uintptr_t>(lse_in) & 3u)))
        return VA3D_ERR_ALIGNMENT;
    if ((rc = check_device()) != VA3D_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const float scale =
        softmax_scale > 0.f ? softmax_scale : static_cast<float>(1.0 / std::sqrt(double(head_dim)));
    SplitScratch none_split = split_scratch(nullptr, 0);
    RopeParams none;
    std::memset(&none, 0, sizeof none);
    const RingMerge m = {first ? 1 : 2, acc, first ? nullptr : lse_in, lse_out};
    return launch_attn(q_rot, k, v, out, nullptr, B * heads, n_rows, n_keys, n_rows, n_keys, 1, false,
                       none, nullptr, scale, none_split, st, nullptr, &m);
}
}  // extern "C"

// ---------------------------------------------------------------------------
// Entry point without a caller workspace, for callers that cannot allocate
// device memory.  Its scratch is this one static device array; every GPU that
// loads the library holds it until the process exits.  In host code the
// array's name is only a host-side stand-in, so the device address is looked
// up with cudaGetSymbolAddress with the device current, and cached.  The
// address belongs to the CUDA context that was current at the lookup, so the
// cache is keyed by that context's unique id (cuCtxGetId): a call under
// another context (a driver-API context of the caller's, or the primary
// context recreated after cudaDeviceReset) looks the address up again.
// Nothing in the scratch needs to start at zero: the table and the rotated
// keys are written before they are read on every call, and the split-tail
// counters behind them are cleared by the table kernel of every call.

static __device__ __align__(256) unsigned char g_noalloc_scratch[VA3D_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mutex;
struct NoallocSlot {
    unsigned long long ctx_id;   // 0: not looked up yet
    void *addr;
};
NoallocSlot g_noalloc_slot[kMaxDevices] = {};

// Unique id of the calling thread's current context; 0 when no context is
// current yet (the runtime creates the primary one on its first use).
int current_context_id(unsigned long long *id) {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    if (get_current == nullptr || get_id == nullptr) return VA3D_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return VA3D_ERR_CUDA;
    *id = 0;
    if (ctx != nullptr && get_id(ctx, id) != CUDA_SUCCESS) return VA3D_ERR_CUDA;
    return VA3D_OK;
}

int noalloc_scratch(void **out) {
    int dev = 0, rc;
    if ((rc = current_device(&dev)) != VA3D_OK) return rc;
    unsigned long long ctx_id = 0;
    if ((rc = current_context_id(&ctx_id)) != VA3D_OK) return rc;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoallocSlot &slot = g_noalloc_slot[dev];
    if (ctx_id == 0 || slot.ctx_id != ctx_id || slot.addr == nullptr) {
        // (the lookup itself makes the primary context current if none was)
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
            return VA3D_ERR_CUDA;
        if (ctx_id == 0 && (rc = current_context_id(&ctx_id)) != VA3D_OK) return rc;
        slot.ctx_id = ctx_id;
        slot.addr = ptr;
    }
    *out = slot.addr;
    return VA3D_OK;
}

}  // namespace

extern "C" int attn3d_full_fwd_noalloc(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v,
                                       va3d_bf16 *o, float *lse, int B, int heads, int N,
                                       int head_dim, const va3d_grid_t *grid, float softmax_scale,
                                       unsigned flags, void *stream) {
    TraceRange trace("va3d.attn3d_full_fwd_noalloc");
    int rc;
    // invalid sizes or grid: report them exactly as the workspace entry does
    if ((rc = check_sizes(B, heads, N, head_dim)) != VA3D_OK) return rc;
    if ((rc = check_grid(grid, N, head_dim)) != VA3D_OK) return rc;
    if (flags & ~static_cast<unsigned>(VA3D_K_ROTATED)) return VA3D_ERR_INVALID;
    // Only the angle table and the rotated keys must fit; the split-tail
    // scratch takes what is left of the array (none: the last wave runs whole).
    if (required_workspace_bytes(B, heads, N, grid, flags) > VA3D_NOALLOC_SCRATCH_BYTES)
        return VA3D_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch)) != VA3D_OK) return rc;
    return full_fwd(q, k, v, o, lse, B, heads, N, head_dim, grid, softmax_scale, flags, scratch,
                    VA3D_NOALLOC_SCRATCH_BYTES, stream, true);
}

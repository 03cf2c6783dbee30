// dm05_suffix_attn.cu -- C ABI of the sm_100a suffix attention: argument
// checks, the split plan, TMA descriptors, the per-device workspace (error
// word) and the launch.  The operation is specified in
// include/dm05_suffix_attn.h.
#include "dm05_suffix_attn.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <thread>
#include <vector>

#include "post_attn_kernels.cuh"
#include "qkv_prologue_kernel.cuh"
#include "suffix_attn_kernel.cuh"

namespace {

constexpr int kTileRows = 64;
constexpr int kStages = 3;
using Layout = dm05::SmemLayout<kTileRows, kStages>;
constexpr size_t kErrBytes = 256;        // error word (padded to one 256-byte segment)
constexpr size_t kPartRowBytes = dm05::kHeadDim * 4 + 16;  // one partial row: D fp32 of O + float4 stats
constexpr int kMaxUnits = 1 << 24;       // B * Hkv
constexpr int kMaxPrefix = 1 << 24;      // P

struct DeviceState {
    uint32_t *err = nullptr;   // device error word
    bool attrs_set = false;
    bool prologue_attrs_set = false;
    bool post_attrs_set = false;
    int num_sms = 0;
    int max_cluster = 0;       // largest cluster size (<= 16) that can be resident
    int active[17] = {};       // active[c]: clusters of c CTAs the device holds at once (0: not allowed)
};

// Partial-result workspace of one (device, stream): concurrent streams never
// share one.  cudaStreamPerThread is a different stream on every thread, so
// for that handle the calling thread is part of the key.
struct StreamWorkspace {
    int dev = -1;
    cudaStream_t stream = nullptr;
    std::thread::id thread;  // default (no thread) unless stream == cudaStreamPerThread
    void *base = nullptr;
    size_t bytes = 0;
};

std::thread::id stream_owner(cudaStream_t stream)
{
    return stream == cudaStreamPerThread ? std::this_thread::get_id() : std::thread::id();
}

std::mutex g_mu;
std::vector<DeviceState> g_dev;
std::vector<StreamWorkspace> g_ws;
std::vector<StreamWorkspace> g_stage;  // device copies of host-buffer calls, per (device, stream)
int g_split_override = 0;
int g_row_block_override = 0;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

auto *kKernel = &dm05::suffix_attn_kernel<kTileRows, kStages>;

// Prologue variants: token tile NT (64 or 128) x ring depth (deep: one CTA per
// SM for grids of about one wave; shallow: two per SM for larger grids), and
// for small grids 64 feature rows per CTA (four CTAs per head).
using PrologueFn = void (*)(CUtensorMap, CUtensorMap, dm05::prologue::Params);
struct PrologueVariant {
    PrologueFn fn;
    int smem;
};
template <int NT, int ST, int MR, int W = 1>
PrologueVariant prologue_variant()
{
    return {&dm05::prologue::qkv_prologue_kernel<NT, ST, MR, W>, dm05::prologue::Smem<NT, ST, MR, W>::kAllocBytes};
}
// the 64-row CTAs in four-chunk stages (one wave, about 192 KB of ring)
template <int NT>
constexpr int wide_stages() { return (192 * 1024) / (4 * (64 * 128 + NT * 128)); }
const PrologueVariant kPrologueVariants[8] = {
    prologue_variant<64, dm05::prologue::deep_stages<64>(), 128>(),
    prologue_variant<64, dm05::prologue::shallow_stages<64>(), 128>(),
    prologue_variant<128, dm05::prologue::deep_stages<128>(), 128>(),
    prologue_variant<128, dm05::prologue::shallow_stages<128>(), 128>(),
    prologue_variant<64, dm05::prologue::deep_stages<64, 64>(), 64>(),
    prologue_variant<128, dm05::prologue::deep_stages<128, 64>(), 64>(),
    prologue_variant<64, wide_stages<64>(), 64, 4>(),
    prologue_variant<128, wide_stages<128>(), 64, 4>(),
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Plan {
    int splits = 1;      // CTAs per (unit, query block): a cluster
    int row_blocks = 1;  // query blocks per unit
    int SQ = 1;          // queries per head per block
};

// Bytes of partial results a call exchanges: [units * row_blocks][splits]
// [G * SQ] rows of D fp32, each followed by a float4 of statistics.
size_t partial_bytes(long long units, const Plan &pl, int G)
{
    return pl.splits > 1 ? static_cast<size_t>(units) * pl.row_blocks * pl.splits * G * pl.SQ * kPartRowBytes : 0;
}

int check_sizes(int B, int Hq, int Hkv, int P, int S, int D)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || P < 0) return DM05_ERR_SHAPE;
    if (Hq % Hkv != 0) return DM05_ERR_SHAPE;
    if (static_cast<long long>(B) * Hkv > kMaxUnits || P > kMaxPrefix) return DM05_ERR_SHAPE;
    if (D != dm05::kHeadDim) return DM05_ERR_UNSUPPORTED;
    if (static_cast<long long>(Hq / Hkv) * S > dm05::kMRows) return DM05_ERR_UNSUPPORTED;
    return DM05_OK;
}

// Work decomposition: CTAs per (sample, KV head) (a cluster that splits its
// key tiles and merges the partial results) and query row blocks per unit
// (each CTA then carries fewer query rows, so fewer partial rows to merge).
// Among the plans whose clusters are all resident at once, the one with the
// lowest estimated cost.

Plan make_plan(int B, int Hq, int Hkv, int P, int S, const DeviceState &ds)
{
    const long long units = static_cast<long long>(B) * Hkv;
    const int G = Hq / Hkv;
    const int tiles = (P + kTileRows - 1) / kTileRows + (S + kTileRows - 1) / kTileRows;
    // every cluster of the call resident at once (no second wave)
    auto fits = [&](int c, long long blocks) {
        if (c == 1) return true;
        return units * blocks * c <= ds.num_sms && units * blocks <= ds.active[c];
    };
    // Estimated cost in microseconds, fitted on B200 measurements of this
    // kernel (base-model chunk, every plan of 1-16 CTAs x 1-5 query blocks,
    // rotating inputs): a split unit costs ~6.4 fixed (launch, first data,
    // merge latency chain), ~1.3 per key tile its slowest CTA streams and
    // ~0.04 per partial row a CTA publishes; an unsplit unit has no merge.
    // Cluster sizes that are not powers of two measured ~1-1.5 slower than
    // the model and are not used.
    auto cost = [&](int c, int sq) {
        const double per_tile = 1.31 * ((tiles + c - 1) / c);
        return c > 1 ? 6.4 + per_tile + 0.04 * G * sq : 3.0 + per_tile;
    };
    const int want_rb = g_row_block_override;
    Plan best;
    best.SQ = S;
    double best_cost = 1e30;
    for (int c = 1; c <= dm05::kMaxSplits; ++c) {
        if (g_split_override > 0 && c != g_split_override) continue;
        if (g_split_override == 0 && ((c & (c - 1)) != 0 || c > ds.max_cluster || !fits(c, 1))) continue;
        // no more CTAs than key tiles: the extra ones only add partials to merge
        // (LIBERO shape, 10 tiles: 8 CTAs 9.87 us, 16 CTAs 9.95 us)
        if (g_split_override == 0 && c > 1 && c > tiles) continue;
        for (int r = 1; r <= 16; ++r) {
            if (c == 1 && r > 1) break;
            const int sq = (S + r - 1) / r;
            if (r > 1 && sq < 8) break;                        // blocks of at least 8 queries per head
            if ((S + sq - 1) / sq != r) continue;              // the same blocks as a smaller r
            if (r > 1 && G * ((sq + 7) / 8 * 8) > dm05::kMRows) continue;
            if (want_rb > 0 ? r != want_rb && !(r == 1 && c == 1) : !fits(c, r)) continue;
            const double t = cost(c, sq);
            if (t < best_cost) {
                best_cost = t;
                best.splits = c;
                best.SQ = sq;
                best.row_blocks = r;
            }
        }
    }
    if (best_cost > 1e29) {  // forced split count that nothing above accepted
        best.splits = g_split_override > 0 ? g_split_override : 1;
        best.row_blocks = 1;
        best.SQ = S;
    }
    if (best.splits > ds.max_cluster) {
        best.splits = ds.max_cluster;
        best.row_blocks = 1;
        best.SQ = S;
    }
    return best;
}

// Work decomposition of a prefix-prefill call: each (sample, KV head)'s P
// query positions are cut into blocks of SQ per head (G * SQ <= 128 MMA
// rows); a block's causal key range is split over `splits` CTAs (a
// cluster, merged as in the suffix call).  The longest block has all
// ceil(P / 64) key tiles; the split count is the cheapest by the same cost
// model among plans whose clusters are all resident at once.
Plan make_prefill_plan(int B, int Hq, int Hkv, int P, const DeviceState &ds)
{
    const long long units = static_cast<long long>(B) * Hkv;
    const int G = Hq / Hkv;
    Plan pl;
    const int sq = (dm05::kMRows / G) / 8 * 8;
    if (P <= sq) {
        pl.SQ = P;  // one block: the whole unit
        pl.row_blocks = 1;
    } else {
        pl.SQ = sq;
        pl.row_blocks = (P + sq - 1) / sq;
    }
    const int tiles = (P + kTileRows - 1) / kTileRows;
    auto cost = [&](int c) {
        double t = 1.2 * ((tiles + c - 1) / c);
        if (c > 1) t += 2.0 + 0.04 * G * pl.SQ;
        return t;
    };
    double best = 1e30;
    for (int c = 1; c <= dm05::kMaxSplits; ++c) {
        if (g_split_override > 0 && c != g_split_override) continue;
        if (g_split_override == 0 && c > 1 &&
            (c > ds.max_cluster || units * pl.row_blocks * c > ds.num_sms ||
             units * pl.row_blocks > ds.active[c]))
            continue;
        if (cost(c) < best) {
            best = cost(c);
            pl.splits = c;
        }
    }
    if (pl.splits > ds.max_cluster) pl.splits = ds.max_cluster;
    return pl;
}

int get_encoder()
{
    if (g_encode) return DM05_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return DM05_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return DM05_OK;
}

// Device state of the current device with kernel attributes set; the error
// word is created only if `allocate` (then `stream` must not be capturing).
// Caller holds g_mu.
int device_state(bool allocate, DeviceState **out, cudaStream_t stream = nullptr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DM05_ERR_CUDA;
    if (dev >= static_cast<int>(g_dev.size())) g_dev.resize(dev + 1);
    DeviceState &ds = g_dev[dev];
    if (!ds.attrs_set) {
        if (cudaDeviceGetAttribute(&ds.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return DM05_ERR_CUDA;
        if (cudaFuncSetAttribute(kKernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout::kAllocBytes) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kKernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
            return DM05_ERR_CUDA;
        // how many clusters of each size the device holds at once with this
        // kernel's footprint (a plan never exceeds it: no second wave)
        ds.max_cluster = 1;
        ds.active[1] = ds.num_sms;
        for (int c = dm05::kMaxSplits; c >= 2; --c) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(c, 1, 1);
            cfg.blockDim = dim3(dm05::kThreads, 1, 1);
            cfg.dynamicSmemBytes = Layout::kAllocBytes;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = c;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kKernel, &cfg) == cudaSuccess && n > 0) {
                ds.active[c] = n;
                if (ds.max_cluster == 1) ds.max_cluster = c;
            } else {
                cudaGetLastError();  // clear a refused size
            }
        }
        ds.attrs_set = true;
    }
    if (allocate && ds.err == nullptr) {
        // cleared on the caller's stream and waited for, so that no kernel on
        // any stream can run before the word holds zero (only ever done
        // outside stream capture)
        void *p = nullptr;
        if (cudaMalloc(&p, kErrBytes) != cudaSuccess) return DM05_ERR_CUDA;
        if (cudaMemsetAsync(p, 0, kErrBytes, stream) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess) {
            cudaFree(p);
            return DM05_ERR_CUDA;
        }
        ds.err = static_cast<uint32_t *>(p);
    }
    *out = &ds;
    return DM05_OK;
}

// Workspace of (current device, stream) with at least `need` bytes.  Grows
// only outside stream capture.  Caller holds g_mu.
int stream_workspace(cudaStream_t stream, size_t need, void **out)
{
    *out = nullptr;
    if (need == 0) return DM05_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DM05_ERR_CUDA;
    const std::thread::id owner = stream_owner(stream);
    StreamWorkspace *w = nullptr;
    for (auto &e : g_ws)
        if (e.dev == dev && e.stream == stream && e.thread == owner) w = &e;
    if (w == nullptr) {
        g_ws.push_back(StreamWorkspace{});
        w = &g_ws.back();
        w->dev = dev;
        w->stream = stream;
        w->thread = owner;
    }
    if (w->bytes < need) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_WORKSPACE;
        if (w->base != nullptr) {
            // cudaFree waits for the device, so no kernel still uses the old buffer
            cudaFree(w->base);
            w->base = nullptr;
            w->bytes = 0;
        }
        void *p = nullptr;
        if (cudaMalloc(&p, need) != cudaSuccess) return DM05_ERR_CUDA;
        w->base = p;
        w->bytes = need;
    }
    *out = w->base;
    return DM05_OK;
}

// A buffer of at least `need` bytes keyed by (current device, stream[, thread
// for cudaStreamPerThread]) in `list`; grows only outside stream capture (a
// smaller existing buffer during capture gives DM05_ERR_WORKSPACE).  Caller
// holds g_mu.
int keyed_buffer(std::vector<StreamWorkspace> &list, cudaStream_t stream, size_t need, void **out)
{
    *out = nullptr;
    if (need == 0) return DM05_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DM05_ERR_CUDA;
    const std::thread::id owner = stream_owner(stream);
    StreamWorkspace *w = nullptr;
    for (auto &e : list)
        if (e.dev == dev && e.stream == stream && e.thread == owner) w = &e;
    if (w == nullptr) {
        list.push_back(StreamWorkspace{});
        w = &list.back();
        w->dev = dev;
        w->stream = stream;
        w->thread = owner;
    }
    if (w->bytes < need) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_WORKSPACE;
        if (w->base != nullptr) {
            cudaFree(w->base);  // waits for the device: no earlier call still uses it
            w->base = nullptr;
            w->bytes = 0;
        }
        void *p = nullptr;
        if (cudaMalloc(&p, need) != cudaSuccess) return DM05_ERR_CUDA;
        w->base = p;
        w->bytes = need;
    }
    *out = w->base;
    return DM05_OK;
}

// Failure-detection self-test: one thread waits, with the attention
// kernel's bounded wait, on a barrier that nothing arrives on (phase 0 of a
// fresh barrier never completes), and records the time-out in the error word
// as the attention kernel does.
__global__ void wait_timeout_selftest_kernel(uint32_t *err, uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        dm05::ptx::mbar_init(&bar, 1);
        dm05::ptx::fence_mbar_init();
        if (!dm05::ptx::mbar_wait(&bar, 0, limit_ns)) atomicOr(err, dm05::kEwTimeout);
    }
}

// Device staging buffer of (current device, stream) for the host-buffer
// entry point, at least `need` bytes.  Caller holds g_mu and has checked that
// the stream is not capturing.
int stream_staging(cudaStream_t stream, size_t need, uint8_t **out)
{
    *out = nullptr;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DM05_ERR_CUDA;
    const std::thread::id owner = stream_owner(stream);
    StreamWorkspace *w = nullptr;
    for (auto &e : g_stage)
        if (e.dev == dev && e.stream == stream && e.thread == owner) w = &e;
    if (w == nullptr) {
        g_stage.push_back(StreamWorkspace{});
        w = &g_stage.back();
        w->dev = dev;
        w->stream = stream;
        w->thread = owner;
    }
    if (w->bytes < need) {
        if (w->base != nullptr) {
            cudaFree(w->base);  // waits for the device: no earlier call still reads it
            w->base = nullptr;
            w->bytes = 0;
        }
        void *p = nullptr;
        if (cudaMalloc(&p, need) != cudaSuccess) return DM05_ERR_CUDA;
        w->base = p;
        w->bytes = need;
    }
    *out = static_cast<uint8_t *>(w->base);
    return DM05_OK;
}

// Places of the tensors in the staging buffer (256-byte aligned offsets).
struct StageLayout {
    size_t q, kp, vp, ks, vs, out, lse, vl, mask, total;
};

StageLayout stage_layout(int B, int Hq, int Hkv, int P, int S, int D)
{
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t row = static_cast<size_t>(D) * 2;
    StageLayout L{};
    size_t o = 0;
    L.q = o;    o += up(static_cast<size_t>(B) * Hq * S * row);
    L.kp = o;   o += up(static_cast<size_t>(B) * Hkv * P * row);
    L.vp = o;   o += up(static_cast<size_t>(B) * Hkv * P * row);
    L.ks = o;   o += up(static_cast<size_t>(B) * Hkv * S * row);
    L.vs = o;   o += up(static_cast<size_t>(B) * Hkv * S * row);
    L.out = o;  o += up(static_cast<size_t>(B) * Hq * S * row);
    L.lse = o;  o += up(static_cast<size_t>(B) * Hq * S * 4);
    L.vl = o;   o += up(static_cast<size_t>(B) * 4);
    L.mask = o; o += up(static_cast<size_t>(B) * P);
    L.total = o;
    return L;
}

// Device address of the host buffer [p, p + n) when the device can store to
// all of it directly (page-locked memory mapped into the device's address
// space, as every cudaHostAlloc / cudaMallocHost buffer is on a 64-bit
// system) and p has the alignment the kernel's stores need; else nullptr.
// Both ends must be mapped and map n - 1 bytes apart, so a buffer that runs
// off its allocation is never written from the device.
void *device_view(void *p, size_t n, size_t align)
{
    if (p == nullptr || n == 0 || reinterpret_cast<uintptr_t>(p) % align != 0) return nullptr;
    uint8_t *first = static_cast<uint8_t *>(p);
    uint8_t *last = first + (n - 1);
    cudaPointerAttributes a{}, z{};
    if (cudaPointerGetAttributes(&a, first) != cudaSuccess || cudaPointerGetAttributes(&z, last) != cudaSuccess) {
        cudaGetLastError();  // an unknown pointer is not an error of the call
        return nullptr;
    }
    if (a.type != cudaMemoryTypeHost || z.type != cudaMemoryTypeHost || a.devicePointer == nullptr ||
        z.devicePointer == nullptr)
        return nullptr;
    if (static_cast<uint8_t *>(z.devicePointer) - static_cast<uint8_t *>(a.devicePointer) !=
        static_cast<ptrdiff_t>(n - 1))
        return nullptr;
    if (reinterpret_cast<uintptr_t>(a.devicePointer) % align != 0) return nullptr;
    return a.devicePointer;
}

// Prefix rows [0, n) of sample b that a host-buffer call copies: the clamped
// valid length, or every row when there is no valid-length array.
int host_rows(const int32_t *valid_len, int b, int P)
{
    if (valid_len == nullptr) return P;
    const int32_t v = valid_len[b];
    return v < 0 ? 0 : v > P ? P : static_cast<int>(v);
}

// bf16 tensor [d2][d1][256] viewed as 4-D [d2][d1][4][64]: the 4 column
// chunks (128 bytes apart) as a dimension inside the row (512 bytes).  A box
// of {64, box1, 4, 1} lands as 4 chunk-major [box1 x 128 B] blocks with
// 128-byte swizzle, the layout the tensor-core descriptors read.
int encode_4d(CUtensorMap *map, const void *base, uint64_t d1, uint64_t d2, uint32_t box1)
{
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(dm05::kChunkElems), d1, static_cast<cuuint64_t>(dm05::kChunks), d2};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(dm05::kHeadDim) * 2, static_cast<cuuint64_t>(dm05::kChunkElems) * 2,
                             d1 * dm05::kHeadDim * 2};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(dm05::kChunkElems), box1, static_cast<cuuint32_t>(dm05::kChunks), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DM05_OK : DM05_ERR_CUDA;
}

// bf16 tensor viewed as [d2][d1][256], loaded in boxes of 64 columns x box1 rows
// with 128-byte swizzle; rows past d1 read as zero.
int encode_3d(CUtensorMap *map, const void *base, uint64_t d1, uint64_t d2, uint32_t box1)
{
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(dm05::kHeadDim), d1, d2};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(dm05::kHeadDim) * 2, d1 * dm05::kHeadDim * 2};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(dm05::kChunkElems), box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DM05_OK : DM05_ERR_CUDA;
}


// bf16 matrix [rows][cols] (cols contiguous) loaded in boxes of 64 columns x
// box_rows rows with 128-byte swizzle; rows past the end read as zero.
int encode_2d(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows, uint32_t box_rows)
{
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DM05_OK : DM05_ERR_CUDA;
}

// Four-chunk ring stages read 256 columns of a row at once (512 contiguous
// bytes) and land them as four chunk-major [box rows][128 B] blocks with
// 128-byte swizzle, the layout the tensor-core descriptors read.
//
// Row-major bf16 [rows][K] viewed as 4-D (64 columns, row, 64-column chunk
// of a 256-column group, group): boxes of 64 x box_rows x 4 x 1.
int encode_wide4(CUtensorMap *map, const void *base, uint64_t rows, uint64_t K, uint32_t box_rows)
{
    cuuint64_t dims[4] = {64, rows, 4, K / 256};
    cuuint64_t strides[3] = {K * 2, 128, 512};
    cuuint32_t box[4] = {64, box_rows, 4, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DM05_OK : DM05_ERR_CUDA;
}

// Row-major bf16 [rows][K] viewed as 5-D (64 columns, row r, pair half h --
// row r or row r + pair --, chunk, group): a box of 64 x box_rows x 2 x 4 x 1
// lands as four chunk-major blocks of [box_rows rows r, then their rows
// r + pair][128 B] (the GEGLU's gate and up rows, the prologue's rotation
// partners).  The row extent is rows - pair, so no box reaches past the matrix.
int encode_pair5(CUtensorMap *map, const void *base, uint64_t rows, uint64_t K, uint64_t pair, uint32_t box_rows)
{
    cuuint64_t dims[5] = {64, rows - pair, 2, 4, K / 256};
    cuuint64_t strides[4] = {K * 2, pair * K * 2, 128, 512};
    cuuint32_t box[5] = {64, box_rows, 2, 4, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DM05_OK : DM05_ERR_CUDA;
}

// Encodes the tensor maps and launches the kernel with plan `pl` on
// `stream`; `err` is the device error word, `part` the partial-result area
// (unused when pl.splits == 1).  Sizes and pointers are already checked.
int launch_attention(const void *q, const void *k_prefix, const void *v_prefix, const int32_t *prefix_valid_len,
                     const uint8_t *prefix_mask, const void *k_suffix, const void *v_suffix, void *out, float *lse,
                     int B, int Hq, int Hkv, int P, int S, int D, const Plan &pl, uint32_t *err, void *part,
                     cudaStream_t stream, bool causal = false, bool prefix_static = false)
{
    const int G = Hq / Hkv;
    const int GS = G * S;
    const long long units = static_cast<long long>(B) * Hkv;
    const long long grid = units * pl.row_blocks * pl.splits;
    if (grid > 0x7fffffffLL) return DM05_ERR_SHAPE;  // more CTAs than one launch can name
    if (pl.splits < 1 || pl.splits > dm05::kMaxSplits) return DM05_ERR_SHAPE;  // the kernel merges only these

    // ---- TMA descriptors (the tensor maps travel as kernel parameters)
    CUtensorMap tm_q, tm_kp, tm_vp, tm_ks, tm_vs;
    // Q: one 128-row box of all four chunks when the block is the whole unit,
    // else one SQ-row box per head and chunk (3-D)
    const int rq = pl.row_blocks == 1
                       ? encode_4d(&tm_q, q, static_cast<uint64_t>(GS), static_cast<uint64_t>(units), dm05::kMRows)
                       : encode_3d(&tm_q, q, static_cast<uint64_t>(GS), static_cast<uint64_t>(units),
                                   static_cast<uint32_t>(pl.SQ));
    if (rq != DM05_OK ||
        encode_4d(&tm_ks, k_suffix, static_cast<uint64_t>(S), static_cast<uint64_t>(units), kTileRows) != DM05_OK ||
        encode_4d(&tm_vs, v_suffix, static_cast<uint64_t>(S), static_cast<uint64_t>(units), kTileRows) != DM05_OK)
        return DM05_ERR_CUDA;
    if (P > 0) {
        if (encode_4d(&tm_kp, k_prefix, static_cast<uint64_t>(P), static_cast<uint64_t>(units), kTileRows) !=
                DM05_OK ||
            encode_4d(&tm_vp, v_prefix, static_cast<uint64_t>(P), static_cast<uint64_t>(units), kTileRows) != DM05_OK)
            return DM05_ERR_CUDA;
    } else {
        tm_kp = tm_ks;  // never read: no prefix tile exists when P == 0
        tm_vp = tm_vs;
    }

    dm05::KernelParams kp;
    kp.valid_len = prefix_valid_len;
    kp.mask = prefix_mask;
    kp.out = static_cast<__nv_bfloat16 *>(out);
    kp.lse = lse;
    kp.err = err;
    kp.part = pl.splits > 1 ? static_cast<float *>(part) : nullptr;
    kp.Hkv = Hkv;
    kp.P = P;
    kp.S = S;
    kp.GS = GS;
    kp.G = G;
    kp.row_blocks = pl.row_blocks;
    kp.SQ = pl.SQ;
    kp.splits = pl.splits;
    kp.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    kp.causal = causal ? 1 : 0;
    kp.prefix_static = prefix_static ? 1 : 0;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(dm05::kThreads, 1, 1);
    cfg.dynamicSmemBytes = Layout::kAllocBytes;
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    int na = 0;
    at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (pl.splits > 1) {
        at[na].id = cudaLaunchAttributeClusterDimension;
        at[na].val.clusterDim.x = static_cast<unsigned>(pl.splits);
        at[na].val.clusterDim.y = 1;
        at[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = at;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, kKernel, tm_q, tm_kp, tm_vp, tm_ks, tm_vs, kp) != cudaSuccess) return DM05_ERR_CUDA;
    return DM05_OK;
}

}  // namespace

extern "C" {

const char *dm05_status_string(int status)
{
    switch (status) {
    case DM05_OK: return "DM05_OK";
    case DM05_ERR_NULL: return "DM05_ERR_NULL: a required pointer is NULL";
    case DM05_ERR_SHAPE: return "DM05_ERR_SHAPE: invalid sizes";
    case DM05_ERR_UNSUPPORTED: return "DM05_ERR_UNSUPPORTED: D must be 256 and (Hq/Hkv)*S at most 128";
    case DM05_ERR_ALIGN: return "DM05_ERR_ALIGN: a bf16 tensor base is not 16-byte aligned";
    case DM05_ERR_WORKSPACE: return "DM05_ERR_WORKSPACE: no workspace on this device while the stream is capturing";
    case DM05_ERR_CUDA: return "DM05_ERR_CUDA: a CUDA call failed";
    default: return "unknown dm05 status";
    }
}

size_t dm05_suffix_attn_workspace_bytes(int B, int Hq, int Hkv, int P, int S, int D)
{
    if (check_sizes(B, Hq, Hkv, P, S, D) != DM05_OK) return 0;
    // the largest split count the library ever uses is 16; row blocks only
    // round each block's queries up (SQ * row_blocks < S + 16)
    Plan worst;
    worst.splits = 16;
    worst.row_blocks = 1;
    worst.SQ = S + 16;  // at most 16 blocks of >= 8 queries
    return kErrBytes + partial_bytes(static_cast<long long>(B) * Hkv, worst, Hq / Hkv);
}

int dm05_set_split_override(int splits_per_head)
{
    if (splits_per_head < 0 || splits_per_head > dm05::kMaxSplits) return DM05_ERR_SHAPE;
    std::lock_guard<std::mutex> lk(g_mu);
    g_split_override = splits_per_head;
    return DM05_OK;
}

int dm05_set_row_block_override(int row_blocks)
{
    if (row_blocks < 0 || row_blocks > 16) return DM05_ERR_SHAPE;
    std::lock_guard<std::mutex> lk(g_mu);
    g_row_block_override = row_blocks;
    return DM05_OK;
}

int dm05_suffix_attn_plan(int B, int Hq, int Hkv, int P, int S, int D, int *splits_per_head, int *tile_rows,
                          int *row_blocks)
{
    int rc = check_sizes(B, Hq, Hkv, P, S, D);
    if (rc != DM05_OK) return rc;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState *ds = nullptr;
    rc = device_state(false, &ds);
    if (rc != DM05_OK) return rc;
    const Plan pl = make_plan(B, Hq, Hkv, P, S, *ds);
    if (splits_per_head) *splits_per_head = pl.splits;
    if (tile_rows) *tile_rows = kTileRows;
    if (row_blocks) *row_blocks = pl.row_blocks;
    return DM05_OK;
}

int dm05_suffix_attn_reserve(int B, int Hq, int Hkv, int P, int S, int D, cudaStream_t stream)
{
    int rc = check_sizes(B, Hq, Hkv, P, S, D);
    if (rc != DM05_OK) return rc;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_WORKSPACE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (get_encoder() != DM05_OK) return DM05_ERR_CUDA;
    DeviceState *ds = nullptr;
    rc = device_state(true, &ds, stream);
    if (rc != DM05_OK) return rc;
    const Plan pl = make_plan(B, Hq, Hkv, P, S, *ds);
    void *ws = nullptr;
    return stream_workspace(stream, partial_bytes(static_cast<long long>(B) * Hkv, pl, Hq / Hkv), &ws);
}

int dm05_suffix_attn(const void *q, const void *k_prefix, const void *v_prefix, const int32_t *prefix_valid_len,
                     const uint8_t *prefix_mask, const void *k_suffix, const void *v_suffix, void *out, float *lse,
                     int B, int Hq, int Hkv, int P, int S, int D, cudaStream_t stream)
{
    return dm05_suffix_attn_ex(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix, v_suffix, out, lse,
                               B, Hq, Hkv, P, S, D, 0u, stream);
}

int dm05_suffix_attn_ex(const void *q, const void *k_prefix, const void *v_prefix, const int32_t *prefix_valid_len,
                        const uint8_t *prefix_mask, const void *k_suffix, const void *v_suffix, void *out,
                        float *lse, int B, int Hq, int Hkv, int P, int S, int D, unsigned flags,
                        cudaStream_t stream)
{
    if ((flags & ~static_cast<unsigned>(DM05_FLAG_PREFIX_STATIC)) != 0) return DM05_ERR_SHAPE;
    // ---- host-side checks; nothing is launched on failure
    if (!q || !k_suffix || !v_suffix || !out) return DM05_ERR_NULL;
    if (P > 0 && (!k_prefix || !v_prefix)) return DM05_ERR_NULL;
    int rc = check_sizes(B, Hq, Hkv, P, S, D);
    if (rc != DM05_OK) return rc;
    if (!aligned16(q) || !aligned16(k_suffix) || !aligned16(v_suffix) || !aligned16(out) ||
        (P > 0 && (!aligned16(k_prefix) || !aligned16(v_prefix))))
        return DM05_ERR_ALIGN;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return DM05_ERR_ALIGN;

    const int G = Hq / Hkv;
    const int units = B * Hkv;

    DeviceState *ds = nullptr;  // points into g_dev: used only while g_mu is held
    uint32_t *err_word = nullptr;
    Plan pl;
    void *part_ws = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (get_encoder() != DM05_OK) return DM05_ERR_CUDA;
        rc = device_state(false, &ds);
        if (rc != DM05_OK) return rc;
        if (ds->err == nullptr) {
            cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
            if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
            if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_WORKSPACE;
            rc = device_state(true, &ds, stream);
            if (rc != DM05_OK) return rc;
        }
        pl = make_plan(B, Hq, Hkv, P, S, *ds);
        err_word = ds->err;
        rc = stream_workspace(stream, partial_bytes(units, pl, G), &part_ws);
        if (rc != DM05_OK) return rc;
    }

    return launch_attention(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix, v_suffix, out, lse, B,
                            Hq, Hkv, P, S, D, pl, err_word, part_ws, stream, false,
                            (flags & DM05_FLAG_PREFIX_STATIC) != 0);
}

int dm05_prefix_prefill_attn(const void *q, const void *k, const void *v, const int32_t *valid_len, void *out,
                             float *lse, int B, int Hq, int Hkv, int P, int D, cudaStream_t stream)
{
    if (!q || !k || !v || !out) return DM05_ERR_NULL;
    if (B < 1 || Hq < 1 || Hkv < 1 || P < 1 || Hq % Hkv != 0) return DM05_ERR_SHAPE;
    if (static_cast<long long>(B) * Hkv > kMaxUnits || P > kMaxPrefix) return DM05_ERR_SHAPE;
    if (D != dm05::kHeadDim || (Hq / Hkv) * 8 > dm05::kMRows) return DM05_ERR_UNSUPPORTED;
    if (static_cast<long long>(Hq / Hkv) * P > 0x7fffffffLL) return DM05_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DM05_ERR_ALIGN;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return DM05_ERR_ALIGN;
    const int G = Hq / Hkv;
    const int units = B * Hkv;
    uint32_t *err_word = nullptr;
    Plan pl;
    void *part_ws = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (get_encoder() != DM05_OK) return DM05_ERR_CUDA;
        DeviceState *ds = nullptr;
        int rc = device_state(false, &ds);
        if (rc != DM05_OK) return rc;
        if (ds->err == nullptr) {
            cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
            if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
            if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_WORKSPACE;
            rc = device_state(true, &ds, stream);
            if (rc != DM05_OK) return rc;
        }
        pl = make_prefill_plan(B, Hq, Hkv, P, *ds);
        err_word = ds->err;
        rc = stream_workspace(stream, partial_bytes(units, pl, G), &part_ws);
        if (rc != DM05_OK) return rc;
    }
    // the queries are the P prefix positions (S = P); no suffix keys exist,
    // so the suffix maps are never read (the prefix K/V stand in for them)
    return launch_attention(q, k, v, valid_len, nullptr, k, v, out, lse, B, Hq, Hkv, P, P, D, pl, err_word, part_ws,
                            stream, true);
}

int dm05_prefix_prefill_reserve(int B, int Hq, int Hkv, int P, int D, cudaStream_t stream)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || P < 1 || Hq % Hkv != 0) return DM05_ERR_SHAPE;
    if (static_cast<long long>(B) * Hkv > kMaxUnits || P > kMaxPrefix) return DM05_ERR_SHAPE;
    if (D != dm05::kHeadDim || (Hq / Hkv) * 8 > dm05::kMRows) return DM05_ERR_UNSUPPORTED;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_WORKSPACE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (get_encoder() != DM05_OK) return DM05_ERR_CUDA;
    DeviceState *ds = nullptr;
    int rc = device_state(true, &ds, stream);
    if (rc != DM05_OK) return rc;
    const Plan pl = make_prefill_plan(B, Hq, Hkv, P, *ds);
    void *ws = nullptr;
    return stream_workspace(stream, partial_bytes(static_cast<long long>(B) * Hkv, pl, Hq / Hkv), &ws);
}

int dm05_prefix_prefill_plan(int B, int Hq, int Hkv, int P, int D, int *splits_per_head, int *query_block,
                             int *row_blocks)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || P < 1 || Hq % Hkv != 0) return DM05_ERR_SHAPE;
    if (D != dm05::kHeadDim || (Hq / Hkv) * 8 > dm05::kMRows) return DM05_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState *ds = nullptr;
    const int rc = device_state(false, &ds);
    if (rc != DM05_OK) return rc;
    const Plan pl = make_prefill_plan(B, Hq, Hkv, P, *ds);
    if (splits_per_head) *splits_per_head = pl.splits;
    if (query_block) *query_block = pl.SQ;
    if (row_blocks) *row_blocks = pl.row_blocks;
    return DM05_OK;
}

int dm05_suffix_qkv_prologue(const void *x, const void *w, const void *q_norm_w, const void *k_norm_w,
                             const int32_t *positions, void *q, void *k, void *v, int B, int S, int H, int Hq,
                             int Hkv, int D, float eps, float theta, cudaStream_t stream)
{
    if (!x || !w || !q_norm_w || !k_norm_w || !positions || !q || !k || !v) return DM05_ERR_NULL;
    if (B < 1 || S < 1 || H < 1 || Hq < 1 || Hkv < 1) return DM05_ERR_SHAPE;
    const long long T = static_cast<long long>(B) * S;
    if (T > (1LL << 24) || H > (1 << 20) || static_cast<long long>(Hq + 2 * Hkv) * D > (1LL << 24))
        return DM05_ERR_SHAPE;
    if (!(eps > 0.0f) || !(theta > 1.0f)) return DM05_ERR_SHAPE;
    if (D != dm05::kHeadDim || H % dm05::prologue::kChunk != 0) return DM05_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(w) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
        (reinterpret_cast<uintptr_t>(q_norm_w) & 1u) || (reinterpret_cast<uintptr_t>(k_norm_w) & 1u) ||
        (reinterpret_cast<uintptr_t>(positions) & 3u))
        return DM05_ERR_ALIGN;
    const bool small = T <= 64;
    uint32_t *err = nullptr;
    int num_sms = 148;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (get_encoder() != DM05_OK) return DM05_ERR_CUDA;
        DeviceState *ds = nullptr;
        int rc = device_state(false, &ds);
        if (rc != DM05_OK) return rc;
        if (ds->err == nullptr || !ds->prologue_attrs_set) {
            cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
            if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
            if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_WORKSPACE;
            rc = device_state(true, &ds, stream);
            if (rc != DM05_OK) return rc;
            for (const PrologueVariant &pv : kPrologueVariants)
                if (cudaFuncSetAttribute(pv.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, pv.smem) != cudaSuccess)
                    return DM05_ERR_CUDA;
            ds->prologue_attrs_set = true;
        }
        err = ds->err;
        num_sms = ds->num_sms;
    }
    const int NT = small ? 64 : 128;
    const long long ctas = static_cast<long long>(2 * (Hq + 2 * Hkv)) * ((T + NT - 1) / NT);
    // 64 feature rows per CTA (four per head) when 128-row CTAs would fill
    // under half the SMs
    const bool mr64 = 2 * ctas <= num_sms;
    // those in four-chunk stages when H is a whole number of 256-column groups
    const bool wide = mr64 && H % 256 == 0;
    const int kq = mr64 ? 4 : 2;
    const PrologueVariant &pv =
        wide   ? kPrologueVariants[small ? 6 : 7]
        : mr64 ? kPrologueVariants[small ? 4 : 5]
               : kPrologueVariants[(small ? 0 : 2) + (ctas > 2LL * num_sms ? 1 : 0)];
    CUtensorMap tm_w, tm_x;
    const uint64_t w_rows = static_cast<uint64_t>(Hq + 2 * Hkv) * D;
    if (wide) {
        // the partner of feature row r is row r + 128 (D = 256)
        if (encode_pair5(&tm_w, w, w_rows, static_cast<uint64_t>(H), 128, 32) != DM05_OK ||
            encode_wide4(&tm_x, x, static_cast<uint64_t>(T), static_cast<uint64_t>(H), static_cast<uint32_t>(NT)) !=
                DM05_OK)
            return DM05_ERR_CUDA;
    } else if (encode_2d(&tm_w, w, static_cast<uint64_t>(H), w_rows, mr64 ? 32 : 64) != DM05_OK ||
               encode_2d(&tm_x, x, static_cast<uint64_t>(H), static_cast<uint64_t>(T), static_cast<uint32_t>(NT)) !=
                   DM05_OK) {
        return DM05_ERR_CUDA;
    }
    dm05::prologue::Params pp;
    pp.qw = static_cast<const __nv_bfloat16 *>(q_norm_w);
    pp.kw = static_cast<const __nv_bfloat16 *>(k_norm_w);
    pp.pos = positions;
    pp.q = static_cast<__nv_bfloat16 *>(q);
    pp.k = static_cast<__nv_bfloat16 *>(k);
    pp.v = static_cast<__nv_bfloat16 *>(v);
    pp.err = err;
    pp.T = static_cast<int>(T);
    pp.S = S;
    pp.H = H;
    pp.Hq = Hq;
    pp.Hkv = Hkv;
    pp.D = D;
    pp.eps = eps;
    pp.log2_theta = std::log2(theta);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(kq * (Hq + 2 * Hkv)), static_cast<unsigned>((T + NT - 1) / NT), 1);
    cfg.blockDim = dim3(dm05::prologue::kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(pv.smem);
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = static_cast<unsigned>(kq);  // the CTAs of a head
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, pv.fn, tm_w, tm_x, pp);
    return e == cudaSuccess ? DM05_OK : DM05_ERR_CUDA;
}


// ---------------------------------------------------------------------------
// Multi-step calls: N suffix-attention calls over one prefix cache captured
// once into a CUDA graph the library owns, then replayed with one launch.
struct dm05_steps_s {
    int dev = -1;
    cudaGraphExec_t exec = nullptr;
    void *workspace = nullptr;  // partial results of split calls, owned by the handle
    int n_steps = 0;
};

int dm05_suffix_attn_steps_create(const dm05_step *steps, int n_steps, const void *k_prefix, const void *v_prefix,
                                  const int32_t *prefix_valid_len, const uint8_t *prefix_mask, int B, int Hq,
                                  int Hkv, int P, int S, int D, unsigned flags, dm05_steps_handle *handle)
{
    if (!handle) return DM05_ERR_NULL;
    *handle = nullptr;
    if (!steps || n_steps < 1 || n_steps > 4096) return n_steps < 1 || n_steps > 4096 ? DM05_ERR_SHAPE : DM05_ERR_NULL;
    if ((flags & ~static_cast<unsigned>(DM05_FLAG_PREFIX_STATIC)) != 0) return DM05_ERR_SHAPE;
    if (P > 0 && (!k_prefix || !v_prefix)) return DM05_ERR_NULL;
    int rc = check_sizes(B, Hq, Hkv, P, S, D);
    if (rc != DM05_OK) return rc;
    if (P > 0 && (!aligned16(k_prefix) || !aligned16(v_prefix))) return DM05_ERR_ALIGN;
    for (int t = 0; t < n_steps; ++t) {
        const dm05_step &st = steps[t];
        if (!st.q || !st.k_suffix || !st.v_suffix || !st.out) return DM05_ERR_NULL;
        if (!aligned16(st.q) || !aligned16(st.k_suffix) || !aligned16(st.v_suffix) || !aligned16(st.out) ||
            (st.lse != nullptr && (reinterpret_cast<uintptr_t>(st.lse) & 3u) != 0))
            return DM05_ERR_ALIGN;
    }
    const int G = Hq / Hkv;
    const int units = B * Hkv;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DM05_ERR_CUDA;
    uint32_t *err_word = nullptr;
    Plan pl;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (get_encoder() != DM05_OK) return DM05_ERR_CUDA;
        DeviceState *ds = nullptr;
        rc = device_state(true, &ds, nullptr);
        if (rc != DM05_OK) return rc;
        pl = make_plan(B, Hq, Hkv, P, S, *ds);
        err_word = ds->err;
    }
    dm05_steps_s *h = new dm05_steps_s();
    h->dev = dev;
    h->n_steps = n_steps;
    const size_t ws_bytes = partial_bytes(units, pl, G);
    if (ws_bytes > 0 && cudaMalloc(&h->workspace, ws_bytes) != cudaSuccess) {
        delete h;
        return DM05_ERR_CUDA;
    }
    // capture the calls, in order, on a private stream
    cudaStream_t cs = nullptr;
    cudaGraph_t graph = nullptr;
    bool ok = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
    int launch_rc = DM05_OK;
    for (int t = 0; ok && t < n_steps && launch_rc == DM05_OK; ++t) {
        const dm05_step &st = steps[t];
        launch_rc = launch_attention(st.q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, st.k_suffix,
                                     st.v_suffix, st.out, st.lse, B, Hq, Hkv, P, S, D, pl, err_word, h->workspace,
                                     cs, false, (flags & DM05_FLAG_PREFIX_STATIC) != 0);
    }
    if (cs != nullptr) {
        cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(cs, &st) == cudaSuccess && st != cudaStreamCaptureStatusNone)
            ok = cudaStreamEndCapture(cs, &graph) == cudaSuccess && ok;
        cudaStreamDestroy(cs);
    }
    if (ok && launch_rc == DM05_OK && graph != nullptr)
        ok = cudaGraphInstantiate(&h->exec, graph, 0) == cudaSuccess;
    if (graph != nullptr) cudaGraphDestroy(graph);
    if (!ok || launch_rc != DM05_OK || h->exec == nullptr) {
        cudaGetLastError();
        if (h->exec) cudaGraphExecDestroy(h->exec);
        if (h->workspace) cudaFree(h->workspace);
        delete h;
        return launch_rc != DM05_OK ? launch_rc : DM05_ERR_CUDA;
    }
    *handle = h;
    return DM05_OK;
}

int dm05_suffix_attn_steps_launch(dm05_steps_handle handle, cudaStream_t stream)
{
    if (!handle) return DM05_ERR_NULL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DM05_ERR_CUDA;
    if (dev != handle->dev) return DM05_ERR_SHAPE;
    return cudaGraphLaunch(handle->exec, stream) == cudaSuccess ? DM05_OK : DM05_ERR_CUDA;
}

int dm05_suffix_attn_steps_destroy(dm05_steps_handle handle)
{
    if (!handle) return DM05_OK;
    int cur = 0;
    const bool have_cur = cudaGetDevice(&cur) == cudaSuccess;
    if (cudaSetDevice(handle->dev) != cudaSuccess) return DM05_ERR_CUDA;
    // no launch of the graph may still be running: wait for the device
    cudaDeviceSynchronize();
    if (handle->exec) cudaGraphExecDestroy(handle->exec);
    if (handle->workspace) cudaFree(handle->workspace);
    delete handle;
    if (have_cur) cudaSetDevice(cur);
    return DM05_OK;
}

int dm05_selftest_wait_timeout(int limit_ms, cudaStream_t stream)
{
    if (limit_ms < 1 || limit_ms > 2000) return DM05_ERR_SHAPE;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_UNSUPPORTED;
    uint32_t *err = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        DeviceState *ds = nullptr;
        const int rc = device_state(true, &ds, stream);
        if (rc != DM05_OK) return rc;
        err = ds->err;
    }
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err, static_cast<uint64_t>(limit_ms) * 1000000ull);
    return cudaGetLastError() == cudaSuccess ? DM05_OK : DM05_ERR_CUDA;
}

int dm05_suffix_attn_host_copy_bytes(const int32_t *prefix_valid_len, int has_prefix_mask, int want_lse, int B,
                                     int Hq, int Hkv, int P, int S, int D, size_t *h2d_bytes, size_t *d2h_bytes)
{
    int rc = check_sizes(B, Hq, Hkv, P, S, D);
    if (rc != DM05_OK) return rc;
    const size_t row = static_cast<size_t>(D) * 2;
    size_t in = static_cast<size_t>(B) * Hq * S * row + 2 * static_cast<size_t>(B) * Hkv * S * row;
    for (int b = 0; b < B; ++b) in += 2 * static_cast<size_t>(Hkv) * host_rows(prefix_valid_len, b, P) * row;
    if (prefix_valid_len != nullptr) in += static_cast<size_t>(B) * 4;
    if (has_prefix_mask) in += static_cast<size_t>(B) * P;
    size_t outb = static_cast<size_t>(B) * Hq * S * row;
    if (want_lse) outb += static_cast<size_t>(B) * Hq * S * 4;
    if (h2d_bytes) *h2d_bytes = in;
    if (d2h_bytes) *d2h_bytes = outb;
    return DM05_OK;
}

int dm05_suffix_attn_host(const void *q, const void *k_prefix, const void *v_prefix, const int32_t *prefix_valid_len,
                          const uint8_t *prefix_mask, const void *k_suffix, const void *v_suffix, void *out,
                          float *lse, int B, int Hq, int Hkv, int P, int S, int D, cudaStream_t stream)
{
    if (!q || !k_suffix || !v_suffix || !out) return DM05_ERR_NULL;
    if (P > 0 && (!k_prefix || !v_prefix)) return DM05_ERR_NULL;
    int rc = check_sizes(B, Hq, Hkv, P, S, D);
    if (rc != DM05_OK) return rc;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_UNSUPPORTED;  // valid lengths are read now

    const StageLayout L = stage_layout(B, Hq, Hkv, P, S, D);
    uint8_t *dv = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        rc = stream_staging(stream, L.total, &dv);
        if (rc != DM05_OK) return rc;
    }
    const size_t row = static_cast<size_t>(D) * 2;
    const size_t q_bytes = static_cast<size_t>(B) * Hq * S * row;
    const size_t suf_bytes = static_cast<size_t>(B) * Hkv * S * row;
    auto h2d = [&](size_t off, const void *src, size_t n) {
        return n == 0 || cudaMemcpyAsync(dv + off, src, n, cudaMemcpyHostToDevice, stream) == cudaSuccess;
    };
    bool ok = h2d(L.q, q, q_bytes) && h2d(L.ks, k_suffix, suf_bytes) && h2d(L.vs, v_suffix, suf_bytes);
    if (ok && prefix_valid_len != nullptr) ok = h2d(L.vl, prefix_valid_len, static_cast<size_t>(B) * 4);
    if (ok && prefix_mask != nullptr) ok = h2d(L.mask, prefix_mask, static_cast<size_t>(B) * P);
    // Prefix K/V: rows [0, clamped valid length) of every (sample, KV head);
    // the kernel reads no row past it.  Runs of samples whose whole bucket is
    // in range are copied as one contiguous block; any other sample as one
    // 2-D copy per tensor (Hkv slabs of n rows at a pitch of P rows).
    const size_t pitch = static_cast<size_t>(P) * row;
    const size_t sample = static_cast<size_t>(Hkv) * pitch;
    const bool pitch_ok = pitch <= static_cast<size_t>(INT32_MAX);
    int run0 = 0;  // first sample of the pending run of whole-bucket samples
    for (int b = 0; ok && P > 0 && b <= B; ++b) {
        const int n = b < B ? host_rows(prefix_valid_len, b, P) : -1;
        if (n == P) continue;
        if (b > run0) {
            const size_t off = static_cast<size_t>(run0) * sample, len = static_cast<size_t>(b - run0) * sample;
            ok = h2d(L.kp + off, static_cast<const uint8_t *>(k_prefix) + off, len) &&
                 h2d(L.vp + off, static_cast<const uint8_t *>(v_prefix) + off, len);
        }
        run0 = b + 1;
        if (!ok || n <= 0) continue;
        const size_t off = static_cast<size_t>(b) * sample, width = static_cast<size_t>(n) * row;
        for (int t = 0; ok && t < 2; ++t) {
            const uint8_t *src = static_cast<const uint8_t *>(t == 0 ? k_prefix : v_prefix) + off;
            uint8_t *dst = dv + (t == 0 ? L.kp : L.vp) + off;
            if (pitch_ok) {
                ok = cudaMemcpy2DAsync(dst, pitch, src, pitch, width, static_cast<size_t>(Hkv),
                                       cudaMemcpyHostToDevice, stream) == cudaSuccess;
            } else {
                for (int h = 0; ok && h < Hkv; ++h)
                    ok = cudaMemcpyAsync(dst + h * pitch, src + h * pitch, width, cudaMemcpyHostToDevice, stream) ==
                         cudaSuccess;
            }
        }
    }
    if (!ok) return DM05_ERR_CUDA;
    // O and the LSE go from the kernel straight into the caller's buffers
    // when the device can address both; otherwise through the staging buffer
    // and a copy back.
    const size_t lse_bytes = static_cast<size_t>(B) * Hq * S * 4;
    void *out_dev = device_view(out, q_bytes, 16);
    void *lse_dev = lse != nullptr ? device_view(lse, lse_bytes, 4) : nullptr;
    const bool direct = out_dev != nullptr && (lse == nullptr || lse_dev != nullptr);
    rc = dm05_suffix_attn(dv + L.q, P > 0 ? dv + L.kp : nullptr, P > 0 ? dv + L.vp : nullptr,
                          prefix_valid_len ? reinterpret_cast<const int32_t *>(dv + L.vl) : nullptr,
                          prefix_mask ? dv + L.mask : nullptr, dv + L.ks, dv + L.vs, direct ? out_dev : dv + L.out,
                          lse == nullptr ? nullptr : static_cast<float *>(direct ? lse_dev : dv + L.lse), B, Hq, Hkv,
                          P, S, D, stream);
    if (rc != DM05_OK || direct) return rc;
    if (cudaMemcpyAsync(out, dv + L.out, q_bytes, cudaMemcpyDeviceToHost, stream) != cudaSuccess) return DM05_ERR_CUDA;
    if (lse != nullptr && cudaMemcpyAsync(lse, dv + L.lse, lse_bytes, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return DM05_ERR_CUDA;
    return DM05_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant.  Its scratch (the kernel's error word) lives in a
// file-scope device array instead of a cudaMalloc'd workspace.  In host code
// the array's name is only a host-side stand-in, never a device address: the
// address the kernel gets comes from cudaGetSymbolAddress, looked up once per
// device with that device current.
namespace {
// [error word: kErrBytes][partial results: the rest]
static __device__ __align__(256) uint32_t g_noalloc_scratch[DM05_NOALLOC_SCRATCH_BYTES / sizeof(uint32_t)];
std::vector<uint32_t *> g_noalloc_addr;  // per device ordinal: device address of g_noalloc_scratch

// Caller holds g_mu.  Looks up (and on first use clears) this device's copy
// of the scratch array.  Allocates nothing.  The clear is enqueued on the
// caller's stream and waited for, so every later kernel on any stream sees a
// zero error word; it runs only outside stream capture.
int noalloc_scratch(cudaStream_t stream, uint32_t **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DM05_ERR_CUDA;
    if (dev >= static_cast<int>(g_noalloc_addr.size())) g_noalloc_addr.resize(dev + 1, nullptr);
    if (g_noalloc_addr[dev] == nullptr) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_WORKSPACE;
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return DM05_ERR_CUDA;
        if (cudaMemsetAsync(ptr, 0, kErrBytes, stream) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess)
            return DM05_ERR_CUDA;
        g_noalloc_addr[dev] = static_cast<uint32_t *>(ptr);
    }
    *out = g_noalloc_addr[dev];
    return DM05_OK;
}

// Device address of this device's scratch array if a call has set it up
// (else nullptr).  Caller holds g_mu.
uint32_t *noalloc_word_if_set_up()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= static_cast<int>(g_noalloc_addr.size())) return nullptr;
    return g_noalloc_addr[dev];
}
}  // namespace

extern "C" {

int dm05_suffix_attn_noalloc(const void *q, const void *k_prefix, const void *v_prefix,
                             const int32_t *prefix_valid_len, const uint8_t *prefix_mask, const void *k_suffix,
                             const void *v_suffix, void *out, float *lse, int B, int Hq, int Hkv, int P, int S,
                             int D, cudaStream_t stream)
{
    if (!q || !k_suffix || !v_suffix || !out) return DM05_ERR_NULL;
    if (P > 0 && (!k_prefix || !v_prefix)) return DM05_ERR_NULL;
    int rc = check_sizes(B, Hq, Hkv, P, S, D);
    if (rc != DM05_OK) return rc;
    if (!aligned16(q) || !aligned16(k_suffix) || !aligned16(v_suffix) || !aligned16(out) ||
        (P > 0 && (!aligned16(k_prefix) || !aligned16(v_prefix))))
        return DM05_ERR_ALIGN;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return DM05_ERR_ALIGN;
    // the error word must fit the fixed array (the partials are sized below)
    if (kErrBytes > DM05_NOALLOC_SCRATCH_BYTES) return DM05_ERR_WORKSPACE;

    const int G = Hq / Hkv;
    const int units = B * Hkv;
    DeviceState *ds = nullptr;
    uint32_t *scratch = nullptr;
    Plan pl;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (get_encoder() != DM05_OK) return DM05_ERR_CUDA;
        rc = device_state(false, &ds);  // kernel attributes only; allocates nothing
        if (rc != DM05_OK) return rc;
        rc = noalloc_scratch(stream, &scratch);
        if (rc != DM05_OK) return rc;
        pl = make_plan(B, Hq, Hkv, P, S, *ds);
        // fewer CTAs per unit until the partial results fit the fixed array
        while (pl.splits > 1 && partial_bytes(units, pl, G) > DM05_NOALLOC_SCRATCH_BYTES - kErrBytes) pl.splits /= 2;
        if (pl.splits == 1) {
            pl.row_blocks = 1;
            pl.SQ = S;
        }
    }

    return launch_attention(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask, k_suffix, v_suffix, out, lse, B,
                            Hq, Hkv, P, S, D, pl, scratch, reinterpret_cast<uint8_t *>(scratch) + kErrBytes, stream);
}

int dm05_get_error_word(cudaStream_t stream, uint32_t *host_word)
{
    if (!host_word) return DM05_ERR_NULL;
    // the word of the allocating entry points and the one in the fixed
    // scratch array of dm05_suffix_attn_noalloc (both, when both exist)
    uint32_t *words[2] = {nullptr, nullptr};
    {
        std::lock_guard<std::mutex> lk(g_mu);
        DeviceState *ds = nullptr;
        int rc = device_state(false, &ds);
        if (rc != DM05_OK) return rc;
        words[0] = ds->err;
        words[1] = noalloc_word_if_set_up();
    }
    *host_word = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return DM05_ERR_CUDA;
    for (uint32_t *w : words) {
        if (w == nullptr) continue;
        uint32_t v = 0;
        if (cudaMemcpyAsync(&v, w, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
            cudaMemsetAsync(w, 0, sizeof(uint32_t), stream) != cudaSuccess ||
            cudaStreamSynchronize(stream) != cudaSuccess)
            return DM05_ERR_CUDA;
        *host_word |= v;
    }
    return DM05_OK;
}

void release_post_buffers();

void dm05_release(void)
{
    std::lock_guard<std::mutex> lk(g_mu);
    int cur = 0;
    bool have_cur = cudaGetDevice(&cur) == cudaSuccess;
    for (size_t d = 0; d < g_dev.size(); ++d) {
        if (g_dev[d].err != nullptr) {
            if (cudaSetDevice(static_cast<int>(d)) == cudaSuccess) cudaFree(g_dev[d].err);
            g_dev[d].err = nullptr;
        }
    }
    for (auto &w : g_ws) {
        if (w.base != nullptr && cudaSetDevice(w.dev) == cudaSuccess) cudaFree(w.base);
    }
    g_ws.clear();
    for (auto &w : g_stage) {
        if (w.base != nullptr && cudaSetDevice(w.dev) == cudaSuccess) cudaFree(w.base);
    }
    g_stage.clear();
    release_post_buffers();
    if (have_cur) cudaSetDevice(cur);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Post-attention block: output projection + residual, Adarms, GEGLU, MLP
// down + gated residual (five launches on the caller's stream).
namespace {

// The output projection reads the attention output in place ([B][Hq][S][D]),
// so its token tiles stay inside one sample (NT tokens of a sample, `tiles`
// per sample).  u and m are plain [B*S][K] matrices: the GEGLU and the MLP
// down run over flat tiles of NTf consecutive tokens that may span samples
// (no padding rows per sample, and 128-token tiles once B*S > 64).
struct PostPlan {
    int NT = 64, tiles = 1, NTf = 64, tiles_f = 1, ks_o = 1, ks_d = 1;
    bool geglu64 = false;  // GEGLU on M = 64 tiles: twice the CTAs when the M = 128 grid is under half the SMs
    bool geglu_wide = false;  // and, within one wave, four-chunk stages (512 contiguous bytes per row)
    size_t off_part_o = 0, off_h1 = 0, off_u = 0, off_m = 0, off_part_d = 0, total = 0;
};

// the largest divisor of `chunks` that is at most `want` (at least 1)
int split_count(int chunks, int want)
{
    int best = 1;
    for (int k = 1; k <= chunks && k <= want; ++k)
        if (chunks % k == 0) best = k;
    return best;
}

PostPlan post_plan(int B, int S, int Hq, int D, int Hd, int F, int num_sms)
{
    PostPlan pl;
    pl.NT = S <= 64 ? 64 : 128;
    pl.tiles = (S + pl.NT - 1) / pl.NT;
    const long long T = static_cast<long long>(B) * S;
    const long long tok_tiles = static_cast<long long>(B) * pl.tiles;
    pl.NTf = T <= 64 ? 64 : 128;
    pl.tiles_f = static_cast<int>((T + pl.NTf - 1) / pl.NTf);
    const long long row_tiles = Hd / 128;
    // spread the two long-K projections over about one wave of CTAs: of
    // one-per-SM CTAs (deep rings) while that needs a split, else of
    // two-per-SM CTAs (shallow rings) when those would add one
    auto splits_for = [&](int chunks, long long tiles) {
        tiles = std::max<long long>(1, tiles);
        long long want = num_sms / tiles;
        if (want < 2) want = (2LL * num_sms) / tiles;
        return split_count(chunks, static_cast<int>(std::max<long long>(1, std::min<long long>(want, 64))));
    };
    pl.ks_o = splits_for(Hq * D / 64, row_tiles * tok_tiles);
    pl.ks_d = splits_for(F / 64, row_tiles * pl.tiles_f);
    pl.geglu64 = 2LL * (F / 64) * pl.tiles_f <= num_sms;
    pl.geglu_wide = pl.geglu64 && (F / 32) * pl.tiles_f <= num_sms && Hd % 256 == 0;
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    size_t o = 0;
    pl.off_part_o = o; o += up(static_cast<size_t>(pl.ks_o) * T * Hd * 4);
    pl.off_h1 = o;     o += up(static_cast<size_t>(T) * Hd * 4);
    pl.off_u = o;      o += up(static_cast<size_t>(T) * Hd * 2);
    pl.off_m = o;      o += up(static_cast<size_t>(T) * F * 2);
    pl.off_part_d = o; o += up(static_cast<size_t>(pl.ks_d) * T * Hd * 4);
    pl.total = o;
    return pl;
}

std::vector<StreamWorkspace> g_post_ws;  // per (device, stream[, thread]) buffers of the post-attention block

// activation viewed as 4-D [B][K / inner][S][inner]; boxes of 64 x NT x 1 x 1
int encode_act(CUtensorMap *map, const void *base, int B, int S, int K, int inner, int NT)
{
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(S),
                          static_cast<cuuint64_t>(K / inner), static_cast<cuuint64_t>(B)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(inner) * 2, static_cast<cuuint64_t>(S) * inner * 2,
                             static_cast<cuuint64_t>(K) * S * 2};
    // [B][S][K] (inner == K): the rows of one sample are K apart, not inner
    if (inner == K) strides[1] = static_cast<cuuint64_t>(S) * K * 2;
    cuuint32_t box[4] = {64, static_cast<cuuint32_t>(NT), 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DM05_OK : DM05_ERR_CUDA;
}

int post_check(const void *attn, const void *h, const void *scale, const void *shift, const void *gate,
               const void *wo, const void *wgu, const void *wd, const void *out, int B, int S, int Hq, int D, int Hd,
               int F)
{
    if (!attn || !h || !scale || !shift || !gate || !wo || !wgu || !wd || !out) return DM05_ERR_NULL;
    if (B < 1 || S < 1 || Hq < 1 || D < 1 || Hd < 1 || F < 1) return DM05_ERR_SHAPE;
    if (static_cast<long long>(B) * S > (1LL << 20) || static_cast<long long>(Hq) * D > (1 << 20) || Hd > (1 << 16) ||
        F > (1 << 20))
        return DM05_ERR_SHAPE;
    if (D % 64 != 0 || Hd % 128 != 0 || F % 64 != 0) return DM05_ERR_UNSUPPORTED;
    for (const void *ptr : {attn, h, wo, wgu, wd, out})
        if (!aligned16(ptr)) return DM05_ERR_ALIGN;
    for (const void *ptr : {scale, shift, gate})
        if (reinterpret_cast<uintptr_t>(ptr) & 7u) return DM05_ERR_ALIGN;  // four bf16 per load
    return DM05_OK;
}

// GEMM variants: epilogue x token tile NT (64 or 128) x ring depth (deep
// for grids of at most one wave, shallow, two CTAs per SM, for larger ones).
using GemmFn = void (*)(CUtensorMap, CUtensorMap, dm05::post::GemmParams);
struct GemmVariant {
    GemmFn fn;
    int smem;
};
template <int NT, int EPI, int ST, int W = 1>
GemmVariant gemm_variant()
{
    return {&dm05::post::gemm_kernel<NT, EPI, ST, W>,
            dm05::post::GemmSmem<NT, ST, EPI == dm05::post::kGeglu64 ? 64 : 128, W>::kAllocBytes};
}
// the M = 64 GEGLU with four-chunk stages (one wave, deep ring)
template <int NT>
GemmVariant geglu64_wide_variant()
{
    constexpr int kSt = (192 * 1024) / (4 * (64 * 128 + NT * 128));
    return gemm_variant<NT, dm05::post::kGeglu64, kSt, 4>();
}
template <int NT, int EPI>
GemmVariant gemm_variant_depth(bool deep)
{
    return deep ? gemm_variant<NT, EPI, dm05::post::deep_stages<NT>()>()
                : gemm_variant<NT, EPI, dm05::post::shallow_stages<NT>()>();
}
GemmVariant gemm_variant_for(int epi, int NT, bool deep)
{
    if (epi == dm05::post::kGeglu64)
        return NT == 64 ? gemm_variant_depth<64, dm05::post::kGeglu64>(deep)
                        : gemm_variant_depth<128, dm05::post::kGeglu64>(deep);
    if (epi == dm05::post::kGeglu)
        return NT == 64 ? gemm_variant_depth<64, dm05::post::kGeglu>(deep)
                        : gemm_variant_depth<128, dm05::post::kGeglu>(deep);
    return NT == 64 ? gemm_variant_depth<64, dm05::post::kPartial>(deep)
                    : gemm_variant_depth<128, dm05::post::kPartial>(deep);
}

int launch_gemm(int epi, int NT, dim3 grid, const CUtensorMap &tw, const CUtensorMap &tx,
                const dm05::post::GemmParams &gp, int num_sms, cudaStream_t stream, bool wide = false)
{
    const long long ctas = static_cast<long long>(grid.x) * grid.y * grid.z;
    // wide: the M = 64 GEGLU in four-chunk stages
    const GemmVariant gv = !wide      ? gemm_variant_for(epi, NT, ctas <= num_sms)
                           : NT == 64 ? geglu64_wide_variant<64>()
                                      : geglu64_wide_variant<128>();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(dm05::post::kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(gv.smem);
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gv.fn, tw, tx, gp) == cudaSuccess ? DM05_OK : DM05_ERR_CUDA;
}

template <class K>
int launch_rows(K kernel, int T, const dm05::post::RowParams &rp, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(T), 1, 1);
    cfg.blockDim = dim3(dm05::post::kRowThreads, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, rp) == cudaSuccess ? DM05_OK : DM05_ERR_CUDA;
}

// Device state with the post-attention kernels' attributes set (once per
// device) and the error word; outside capture only.  Caller holds g_mu.
int post_device_state(cudaStream_t stream, DeviceState **out)
{
    DeviceState *ds = nullptr;
    int rc = device_state(false, &ds);
    if (rc != DM05_OK) return rc;
    if (ds->err == nullptr || !ds->post_attrs_set) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return DM05_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone) return DM05_ERR_WORKSPACE;
        rc = device_state(true, &ds, stream);
        if (rc != DM05_OK) return rc;
        for (int v = 0; v < 14; ++v) {
            const GemmVariant gv = v < 12    ? gemm_variant_for(v % 3, (v / 3) & 1 ? 128 : 64, (v / 6) != 0)
                                 : v == 12 ? geglu64_wide_variant<64>()
                                           : geglu64_wide_variant<128>();
            if (cudaFuncSetAttribute(gv.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, gv.smem) != cudaSuccess)
                return DM05_ERR_CUDA;
        }
        ds->post_attrs_set = true;
    }
    *out = ds;
    return DM05_OK;
}

}  // namespace

extern "C" {

int dm05_post_attention_reserve(int B, int S, int Hq, int D, int Hd, int F, cudaStream_t stream)
{
    if (B < 1 || S < 1 || Hq < 1 || D < 1 || Hd < 1 || F < 1) return DM05_ERR_SHAPE;
    if (D % 64 != 0 || Hd % 128 != 0 || F % 64 != 0) return DM05_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (get_encoder() != DM05_OK) return DM05_ERR_CUDA;
    DeviceState *ds = nullptr;
    int rc = post_device_state(stream, &ds);
    if (rc != DM05_OK) return rc;
    const PostPlan pl = post_plan(B, S, Hq, D, Hd, F, ds->num_sms);
    void *ws = nullptr;
    return keyed_buffer(g_post_ws, stream, pl.total, &ws);
}

int dm05_post_attention(const void *attn, const void *h, const void *scale, const void *shift, const void *gate,
                        const void *wo, const void *wgu, const void *wd, void *out, int B, int S, int Hq, int D,
                        int Hd, int F, float eps, cudaStream_t stream)
{
    int rc = post_check(attn, h, scale, shift, gate, wo, wgu, wd, out, B, S, Hq, D, Hd, F);
    if (rc != DM05_OK) return rc;
    if (!(eps > 0.0f)) return DM05_ERR_SHAPE;
    const int T = B * S;
    PostPlan pl;
    int num_sms = 148;
    uint32_t *err = nullptr;
    uint8_t *ws = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (get_encoder() != DM05_OK) return DM05_ERR_CUDA;
        DeviceState *ds = nullptr;
        rc = post_device_state(stream, &ds);
        if (rc != DM05_OK) return rc;
        pl = post_plan(B, S, Hq, D, Hd, F, ds->num_sms);
        num_sms = ds->num_sms;
        err = ds->err;
        void *p = nullptr;
        rc = keyed_buffer(g_post_ws, stream, pl.total, &p);
        if (rc != DM05_OK) return rc;
        ws = static_cast<uint8_t *>(p);
    }
    float *part_o = reinterpret_cast<float *>(ws + pl.off_part_o);
    float *h1 = reinterpret_cast<float *>(ws + pl.off_h1);
    __nv_bfloat16 *u = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_u);
    __nv_bfloat16 *m = reinterpret_cast<__nv_bfloat16 *>(ws + pl.off_m);
    float *part_d = reinterpret_cast<float *>(ws + pl.off_part_d);

    CUtensorMap tw_o, tw_gu, tw_d, tx_a, tx_u, tx_m;
    const int A = Hq * D;
    if (encode_2d(&tw_o, wo, static_cast<uint64_t>(A), static_cast<uint64_t>(Hd), 64) != DM05_OK ||
        (pl.geglu_wide ? encode_pair5(&tw_gu, wgu, static_cast<uint64_t>(2) * F, static_cast<uint64_t>(Hd),
                                      static_cast<uint64_t>(F), 32)
                       : encode_2d(&tw_gu, wgu, static_cast<uint64_t>(Hd), static_cast<uint64_t>(2) * F,
                                   pl.geglu64 ? 32 : 64)) != DM05_OK ||
        encode_2d(&tw_d, wd, static_cast<uint64_t>(F), static_cast<uint64_t>(Hd), 64) != DM05_OK ||
        encode_act(&tx_a, attn, B, S, A, D, pl.NT) != DM05_OK ||
        (pl.geglu_wide ? encode_wide4(&tx_u, u, static_cast<uint64_t>(T), static_cast<uint64_t>(Hd),
                                      static_cast<uint32_t>(pl.NTf))
                       : encode_act(&tx_u, u, 1, T, Hd, Hd, pl.NTf)) != DM05_OK ||
        encode_act(&tx_m, m, 1, T, F, F, pl.NTf) != DM05_OK)
        return DM05_ERR_CUDA;

    dm05::post::GemmParams gp{};
    gp.err = err;
    gp.T = T;
    gp.S = S;
    gp.tiles_per_sample = pl.tiles;
    const unsigned tok_tiles = static_cast<unsigned>(B * pl.tiles);
    // 1. output projection: partial sums over ks_o K ranges
    gp.part = part_o;
    gp.N_rows = Hd;
    gp.xk_inner = D;
    gp.chunks_per_split = A / 64 / pl.ks_o;
    rc = launch_gemm(dm05::post::kPartial, pl.NT, dim3(Hd / 128, tok_tiles, pl.ks_o), tw_o, tx_a, gp, num_sms, stream);
    if (rc != DM05_OK) return rc;
    // 2. residual, Adarms
    dm05::post::RowParams rp{};
    rp.part = part_o;
    rp.splits = pl.ks_o;
    rp.h = static_cast<const __nv_bfloat16 *>(h);
    rp.scale = static_cast<const __nv_bfloat16 *>(scale);
    rp.shift = static_cast<const __nv_bfloat16 *>(shift);
    rp.gate = static_cast<const __nv_bfloat16 *>(gate);
    rp.h1 = h1;
    rp.u = u;
    rp.out = static_cast<__nv_bfloat16 *>(out);
    rp.T = T;
    rp.S = S;
    rp.Hd = Hd;
    rp.eps = eps;
    rc = launch_rows(dm05::post::adarms_rows, T, rp, stream);
    if (rc != DM05_OK) return rc;
    // 3. GEGLU gate-up, over flat token tiles (one "sample" of T tokens)
    gp.part = nullptr;
    gp.m = m;
    gp.F = F;
    gp.xk_inner = Hd;
    gp.chunks_per_split = Hd / 64;
    gp.S = T;
    gp.tiles_per_sample = pl.tiles_f;
    const unsigned flat_tiles = static_cast<unsigned>(pl.tiles_f);
    if (pl.geglu64)
        rc = launch_gemm(dm05::post::kGeglu64, pl.NTf, dim3(F / 32, flat_tiles, 1), tw_gu, tx_u, gp, num_sms, stream,
                         pl.geglu_wide);
    else
        rc = launch_gemm(dm05::post::kGeglu, pl.NTf, dim3(F / 64, flat_tiles, 1), tw_gu, tx_u, gp, num_sms, stream);
    if (rc != DM05_OK) return rc;
    // 4. MLP down: partial sums over ks_d K ranges
    gp.part = part_d;
    gp.m = nullptr;
    gp.N_rows = Hd;
    gp.xk_inner = F;
    gp.chunks_per_split = F / 64 / pl.ks_d;
    rc = launch_gemm(dm05::post::kPartial, pl.NTf, dim3(Hd / 128, flat_tiles, pl.ks_d), tw_d, tx_m, gp, num_sms, stream);
    if (rc != DM05_OK) return rc;
    // 5. gated residual
    rp.part = part_d;
    rp.splits = pl.ks_d;
    return launch_rows(dm05::post::gated_residual_rows, T, rp, stream);
}

}  // extern "C"

// Frees the post-attention block's buffers (called by dm05_release with g_mu held).
void release_post_buffers()
{
    for (auto &w : g_post_ws) {
        if (w.base != nullptr && cudaSetDevice(w.dev) == cudaSuccess) cudaFree(w.base);
    }
    g_post_ws.clear();
}

// suffix_attn_kernel.cuh -- sm_100a kernel of the DM0.5 action-expert
// (suffix) attention.
//
// What it computes (page "TensorRT+Triton+FlexAttention: OpenDM VLA
// 快速推理加速栈深度剖析", section 2.2): logits of the suffix queries against
// the prefix KV cache and the suffix K/V at once under the prefix-visibility
// mask, an online softmax, and the value-weighted sum; 8 query heads over 4
// KV heads (GQA), head_dim 256 (same section's shape table).
//
// Design (one CTA = one slice of the key rows of one (sample, KV head) unit):
//   * The query heads of a GQA group form one MMA A operand: M = G*S <= 128
//     rows (padded to 128 by TMA zero fill), K = D = 256, so every K/V tile
//     is loaded once and used by both heads.  When a unit is split over a
//     cluster and SMs are left over, its S queries are also split into
//     row blocks (each CTA then holds both heads' SQ queries of one block),
//     which halves the partial results each CTA must merge.
//   * Key rows are a list of 64-row tiles: the S suffix rows, then the
//     prefix rows [0, valid_len).  The CTAs of one unit split that list
//     evenly (the split depends on valid_len, read on the device, so a
//     captured graph stays valid for any valid_len).  Each CTA requests its
//     first tile's K/V before the valid_len read returns (the tile it would
//     get if valid_len were P, which is nearly always the same one).
//   * Warp roles: warp 8 issues TMA loads (Q once, then a ring of K and V
//     tiles); warp 9 allocates TMEM, copies Q from shared memory into TMEM
//     (where it stays, so its shared memory becomes the ring's third
//     stage) and issues tcgen05 MMAs from one thread; warps 0-7 run the
//     softmax: warps w and w+4 share TMEM lane quarter w (32 query rows) and
//     each takes half of every tile's columns.
//   * S = Q K^T (A = Q from TMEM, B = the K tile in shared memory) goes to
//     TMEM (two rotating buffers).  Each softmax thread reads half of its
//     row with tcgen05.ld, applies the mask, combines its half's maximum
//     with the partner warp's (shared memory and a bounded pair barrier),
//     computes p = 2^(s * scale - m) with paired fp32 arithmetic, keeps the
//     running max m and its half of the sums, and writes P (bf16) back into
//     the same TMEM columns.  O += P V is a tcgen05 MMA with A = P read from
//     TMEM and B = the V tile in shared memory (MN-major).  O (128 x 256
//     fp32) lives in TMEM for the whole pass.
//   * The running max is updated lazily: O and l are rescaled only when the
//     tile max exceeds the current max by more than 2^8 (exact: O and l use
//     the same stale max, and p <= 2^8 stays well inside fp32/bf16 range).
//   * Splits of one unit form a thread-block cluster (the hardware barrier
//     that orders the merge, and a guarantee that all splits are resident).
//     Each CTA publishes its unnormalised partial O with its per-row
//     (m, l, l_hat) to a workspace in L2 (one 1040-byte bulk TMA store per
//     row); after one cluster barrier CTA r loads rows [r*GS/C, (r+1)*GS/C)
//     of every partial with one bulk copy per partial and combines them by
//     the log-sum-exp rule.  (Distributed shared memory, as loads and as
//     bulk pushes, and plain stores and loads through L2 were measured
//     slower for this traffic.)
//   * Every wait is bounded (2 s): on time-out the kernel records
//     DM05_EW_WAIT_TIMEOUT in the error word, drains its own copies and MMAs
//     (again bounded), frees TMEM and returns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace dm05 {

// Phase time stamps for timeline studies: compiled in only when DM05_TRACE
// is defined (never in the library build); each records the SM clock (or,
// for the first and last slot, the global timer) of one CTA's phase boundary.
#ifdef DM05_TRACE
__device__ unsigned long long g_dm05_trace[4096][16];
__device__ unsigned long long g_dm05_tile_trace[4096][8][24];  // per tile: K full, QK issued, S seen, P ready, K requested, PV issued, QK start, PV start
#define DM05_TRACE_CLOCK(slot)                                                      \
    do {                                                                            \
        if (blockIdx.x < 4096) g_dm05_trace[blockIdx.x][slot] = clock64();          \
    } while (0)
#define DM05_TRACE_GTIME(slot)                                                      \
    do {                                                                            \
        if (blockIdx.x < 4096) g_dm05_trace[blockIdx.x][slot] = ptx::globaltimer_ns(); \
    } while (0)
#define DM05_TRACE_TILE(ev, t)                                                              \
    do {                                                                                    \
        if (blockIdx.x < 4096 && (t) < 24) g_dm05_tile_trace[blockIdx.x][ev][t] = clock64(); \
    } while (0)
#else
#define DM05_TRACE_CLOCK(slot) \
    do {                       \
    } while (0)
#define DM05_TRACE_GTIME(slot) \
    do {                       \
    } while (0)
#define DM05_TRACE_TILE(ev, t) \
    do {                       \
    } while (0)
#endif

constexpr int kHeadDim = 256;
constexpr int kMRows = 128;                       // MMA M: query rows (padded)
constexpr int kChunkElems = 64;                   // bf16 per 128-byte swizzle row
constexpr int kChunks = kHeadDim / kChunkElems;   // 4 column chunks of a row
constexpr int kSoftmaxWarps = 8;   // 2 per TMEM lane quarter: rows x column halves
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;                    // O: columns [0, 256)
constexpr uint32_t kTmemQ = 256;                  // Q as bf16 pairs: columns [256, 384)
constexpr uint32_t kTmemS = 384;                  // S/P buffers: [384, 384 + kSBufs*NT)
constexpr int kSBufs = 2;                         // S/P TMEM buffers in flight
constexpr int kMaxSplits = 16;                    // CTAs per split cluster (the hardware's largest cluster)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr float kRescaleThreshold = 8.0f;         // log2 units: p <= 2^8 between rescales
constexpr uint32_t kEwClamped = 0x1u;
constexpr uint32_t kEwTimeout = 0x2u;
constexpr uint32_t kEwBadSplit = 0x4u;

struct KernelParams {
    const int32_t *valid_len;  // [B] or nullptr
    const uint8_t *mask;       // [B, P] or nullptr
    __nv_bfloat16 *out;        // [B*Hkv, GS, D]
    float *lse;                // [B*Hkv, GS] or nullptr
    uint32_t *err;             // device error word
    float *part;               // splits > 1: partial rows [units*row_blocks][splits][G*SQ], each D fp32 + {m, l, l_hat, 0}
    int Hkv, P, S, GS;         // GS = (Hq / Hkv) * S query rows of a unit
    int G;                     // query heads per KV head
    int row_blocks;            // query blocks per unit (1: all S queries in one CTA)
    int SQ;                    // queries per head per block (S when row_blocks == 1)
    int splits;                // CTAs per (unit, query block): the cluster size
    float scale_log2;          // log2(e) / sqrt(D)
    int prefix_static;         // 1: the preceding grid writes neither the prefix K/V, valid_len nor
                               // the mask, so they may be read before it completes
    int causal;                // 0: suffix attention; 1: prefix prefill (queries are the P prefix
                               // positions, S == P, no suffix keys, key j visible to query i iff j <= i)
};

template <int NT, int STAGES>
struct SmemLayout {
    static_assert(NT % 32 == 0 && NT >= 32 && kTmemS + kSBufs * NT <= kTmemCols, "tile rows");
    static constexpr int kQChunkBytes = kMRows * 128;                 // 16 KB
    static constexpr int kQBytes = kChunks * kQChunkBytes;            // 64 KB
    static constexpr int kTileChunkBytes = NT * 128;
    static constexpr int kTileBytes = kChunks * kTileChunkBytes;      // NT * 512
    // ring stage s: the K tile at s * kStageBytes, the V tile right after it
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kDataEnd = STAGES * kStageBytes;
    // Q lands in the last stage and stays there until it is copied to TMEM
    static constexpr int kQOff = (STAGES - 1) * kStageBytes;
    static_assert(kStageBytes >= kQBytes, "Q must fit in one ring stage");
    // barriers
    static constexpr int kBarQFull = 0;
    static constexpr int kBarQFree = kBarQFull + 1;         // Q copied to TMEM: its stage may be reused
    static constexpr int kBarKFull = kBarQFree + 1;
    static constexpr int kBarKEmpty = kBarKFull + STAGES;
    static constexpr int kBarVFull = kBarKEmpty + STAGES;
    static constexpr int kBarVEmpty = kBarVFull + STAGES;
    static constexpr int kBarSFull = kBarVEmpty + STAGES;    // per S/P buffer
    static constexpr int kBarPReady = kBarSFull + kSBufs;    // per S/P buffer
    static constexpr int kBarPFree = kBarPReady + kSBufs;    // per S/P buffer
    static constexpr int kBarMmaFinal = kBarPFree + kSBufs;
    static constexpr int kBarMerge = kBarMmaFinal + 1;
    static constexpr int kBarPair = kBarMerge + 1;          // per TMEM lane quarter: its 2 softmax warps
    static constexpr int kNumBars = kBarPair + 4;
    static constexpr int kBarOff = kDataEnd;
    static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
    // softmax half exchange: row maxima [2][2][128], sums [2][128] x 2
    static constexpr int kXchgOff = (kTmemSlotOff + 16 + 15) / 16 * 16;
    static constexpr int kEnd = kXchgOff + (4 + 2 + 2) * kMRows * 4;
    static constexpr int kAllocBytes = kEnd + 1024;                  // slack for 1 KB alignment
    // The merge stages up to 128 rows at kStageStride bytes, then receives
    // at most (128 + 16) rows of 1 KB, both inside the data region.
    static constexpr int kStageStride = kHeadDim * 4 + 16;           // padded: conflict-free row writes
    static_assert(kDataEnd >= kMRows * kStageStride, "staging area must fit in the data region");
    static_assert(kDataEnd >= (kMRows + 16) * kStageStride, "receive area must fit in the data region");
};

struct TileInfo {
    bool prefix;
    int row0;     // first key row (prefix row or suffix row index)
    int n_valid;  // rows of the tile that are in range
};

// Tile g of a unit's key list: the TS suffix tiles first, then the prefix
// tiles of [0, vl).  A tile's rows (row0) do not depend on vl, only how many
// of them are valid.
template <int NT>
__device__ __forceinline__ TileInfo tile_of(int g, int TS, int vl, int S)
{
    TileInfo ti;
    if (g < TS) {
        ti.prefix = false;
        ti.row0 = g * NT;
        ti.n_valid = min(NT, S - ti.row0);
    } else {
        ti.prefix = true;
        ti.row0 = (g - TS) * NT;
        ti.n_valid = min(NT, vl - ti.row0);
    }
    return ti;
}

// All lanes of a warp wait on the barrier; the result is made warp-uniform.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity)
{
    bool ok = ptx::mbar_wait(bar, parity, kWaitLimitNs);
    return __all_sync(0xffffffffu, ok);
}

// Two probabilities rounded to bf16 (the MMA operand), low half = lo.  The
// rounded values are summed too: they normalise O, so that O is an exact
// convex combination of V rows with the weights the MMA used; the fp32
// values give the LSE.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// out row of compact row k = h * nq + j of a query block: head h, query q0 + j
__device__ __forceinline__ size_t block_out_row(size_t unit_row0, int k, int nq, int S, int q0)
{
    const int h = k / nq;
    return unit_row0 + static_cast<size_t>(h) * S + q0 + (k - h * nq);
}

// Merge of the nr partial rows this CTA owns (rows whose query index within
// the block is jlim or more are not written).  Partial c's row rr sits at
// recv + (c * nr + rr) * kStageStride: D fp32 of unnormalised O, then
// {m, l, l_hat, 0}.  By the log-sum-exp rule
//   M = max_c m_c,  w_c = 2^(m_c - M),  LH = sum_c l_hat_c w_c,  L = sum_c l_c w_c,
//   out = sum_c (w_c / LH) O_c,  lse = (M + log2 L) ln 2,
// where a partial without visible keys (l_hat == 0) gets no weight.
// Pass 1 (merge_weights): each row takes a segment of W lanes (W = C rounded
// up to a power of two), lane c of the segment holding partial c's
// statistics, so a warp reduces 32 / W rows at once with segment-wide
// shuffles; the row's normalised weights w_c / LH replace the unused fourth
// statistic of each partial row, the LSE is written, and orow[rr] receives
// the row's output row (or -1 when the row is not written), so that pass 2
// does no index arithmetic.
template <class L>
__device__ __forceinline__ void merge_weights(uint8_t *recv, int C, int nr, float *lse, size_t unit_row0, int k_lo,
                                              int nq, int S, int q0, int jlim, long long *orow)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int W = 1;
    while (W < C) W <<= 1;  // C <= 16, so W <= 16
    const int per_warp = 32 / W;
    const int seg = lane / W, c = lane - seg * W;
    const size_t cstride = static_cast<size_t>(nr) * L::kStageStride;
    // every lane of the warp runs the same number of rounds (shuffles need them all)
    for (int base = warp * per_warp; base < nr; base += (kThreads / 32) * per_warp) {
        const int rr = base + seg;
        const bool row_ok = rr < nr;
        float4 st = make_float4(-INFINITY, 0.f, 0.f, 0.f);
        float *slot = nullptr;
        if (row_ok && c < C) {
            slot = reinterpret_cast<float *>(recv + c * cstride + rr * L::kStageStride + kHeadDim * 4);
            st = *reinterpret_cast<const float4 *>(slot);
        }
        const bool has = st.z > 0.0f;
        float M = has ? st.x : -INFINITY;
        for (int o = W >> 1; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o, W));
        const float w = has ? ptx::ex2(st.x - M) : 0.0f;
        float LH = st.z * w, Ls = st.y * w;
        for (int o = W >> 1; o > 0; o >>= 1) {
            LH += __shfl_xor_sync(0xffffffffu, LH, o, W);
            Ls += __shfl_xor_sync(0xffffffffu, Ls, o, W);
        }
        if (slot != nullptr) slot[3] = w / LH;
        if (row_ok && c == 0) {
            const bool written = (k_lo + rr) % nq < jlim;
            const size_t o = block_out_row(unit_row0, k_lo + rr, nq, S, q0);
            orow[rr] = written ? static_cast<long long>(o) : -1;
            if (written && lse != nullptr) lse[o] = (M + ptx::lg2(Ls)) * 0.69314718055994531f;
        }
    }
}

// Pass 2 (after a CTA barrier): one item per (row, 4-column quad):
// out = sum_c wn_c O_c, two partials' loads in flight at a time.
template <class L>
__device__ __forceinline__ void merge_rows(const uint8_t *recv, int C, int nr, __nv_bfloat16 *out,
                                           const long long *orow)
{
    const int items = nr * (kHeadDim / 4);
    const size_t cstride = static_cast<size_t>(nr) * L::kStageStride;
    int trace_n = 0;
    for (int i = threadIdx.x; i < items; i += kThreads) {
        const int rr = i / (kHeadDim / 4), ch = i - rr * (kHeadDim / 4);
        if (threadIdx.x == 0 && trace_n < 2) DM05_TRACE_TILE(4 + trace_n, 22);
        ++trace_n;
        const long long o = orow[rr];
        if (o < 0) continue;
        const uint8_t *row = recv + rr * L::kStageStride;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        // a partial without keys (weight 0) may hold anything, NaN included
        auto add = [&](float w, const float4 &v) {
            const bool use = w != 0.0f;
            const float ww = use ? w : 0.0f;
            acc.x = fmaf(ww, use ? v.x : 0.0f, acc.x);
            acc.y = fmaf(ww, use ? v.y : 0.0f, acc.y);
            acc.z = fmaf(ww, use ? v.z : 0.0f, acc.z);
            acc.w = fmaf(ww, use ? v.w : 0.0f, acc.w);
        };
        int c = 0;
        for (; c + 2 <= C; c += 2) {
            const uint8_t *r0 = row + c * cstride, *r1 = r0 + cstride;
            const float w0 = *reinterpret_cast<const float *>(r0 + kHeadDim * 4 + 12);
            const float w1 = *reinterpret_cast<const float *>(r1 + kHeadDim * 4 + 12);
            const float4 v0 = *reinterpret_cast<const float4 *>(r0 + ch * 16);
            const float4 v1 = *reinterpret_cast<const float4 *>(r1 + ch * 16);
            add(w0, v0);
            add(w1, v1);
        }
        if (c < C) {
            const uint8_t *r0 = row + c * cstride;
            add(*reinterpret_cast<const float *>(r0 + kHeadDim * 4 + 12), *reinterpret_cast<const float4 *>(r0 + ch * 16));
        }
        __nv_bfloat162 h0 = __floats2bfloat162_rn(acc.x, acc.y);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(acc.z, acc.w);
        *reinterpret_cast<uint2 *>(out + static_cast<size_t>(o) * kHeadDim + ch * 4) =
            make_uint2(*reinterpret_cast<uint32_t *>(&h0), *reinterpret_cast<uint32_t *>(&h1));
    }
}

template <int NT, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    suffix_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kp,
                       const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ CUtensorMap tm_ks,
                       const __grid_constant__ CUtensorMap tm_vs, const KernelParams p)
{
    using L = SmemLayout<NT, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kTmemSlotOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int C = p.splits;
    const int cl = blockIdx.x / C;  // cluster: one query block of one unit
    const int rank = blockIdx.x - cl * C;
    const int unit = cl / p.row_blocks;
    const int rb = cl - unit * p.row_blocks;
    const int b = unit / p.Hkv;
    // TMEM row m <-> head m / rph, query q0 + m % rph (valid if that is < nq);
    // compact row k = head * nq + (m % rph) indexes the valid rows.
    const int q0 = rb * p.SQ;
    const int nq = min(p.SQ, p.S - q0);
    const int rph = p.row_blocks == 1 ? p.S : (p.SQ + 7) / 8 * 8;
    const int NR = p.G * nq;
    const size_t unit_row0 = static_cast<size_t>(unit) * p.GS;

    // ---- set-up that reads no input (overlaps the previous kernel under PDL)
    if (threadIdx.x == 0) {
        DM05_TRACE_GTIME(0);
        DM05_TRACE_CLOCK(1);
    }
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bars[L::kBarQFull], 1);
        ptx::mbar_init(&bars[L::kBarQFree], 1);
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&bars[L::kBarKFull + s], 1);
            ptx::mbar_init(&bars[L::kBarKEmpty + s], 1);
            ptx::mbar_init(&bars[L::kBarVFull + s], 1);
            ptx::mbar_init(&bars[L::kBarVEmpty + s], 1);
        }
        for (int i = 0; i < kSBufs; ++i) {
            ptx::mbar_init(&bars[L::kBarSFull + i], 1);
            ptx::mbar_init(&bars[L::kBarPReady + i], kSoftmaxWarps * 32);
            ptx::mbar_init(&bars[L::kBarPFree + i], 1);
        }
        ptx::mbar_init(&bars[L::kBarMmaFinal], 1);
        ptx::mbar_init(&bars[L::kBarMerge], 1);
        for (int i = 0; i < 4; ++i) ptx::mbar_init(&bars[L::kBarPair + i], 64);
        ptx::fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_kp);
        ptx::prefetch_tensormap(&tm_vp);
        ptx::prefetch_tensormap(&tm_ks);
        ptx::prefetch_tensormap(&tm_vs);
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::griddep_launch_dependents();
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // ---- from here on inputs are read: wait for the preceding grid.  With
    // a static prefix the TMA producer first requests the prefix tiles of its
    // first ring slots (the preceding grid does not write them), and waits
    // just before it needs Q or a suffix tile.
    const bool early = p.prefix_static && warp == kProducerWarp && lane == 0;
    if (!early) ptx::griddep_wait();
    if (threadIdx.x == 0) DM05_TRACE_CLOCK(2);

    uint8_t *sQ = smem + L::kQOff;
    auto sK = [&](int s) { return smem + s * L::kStageBytes; };
    auto sV = [&](int s) { return smem + s * L::kStageBytes + L::kTileBytes; };
    // This CTA's first tile if valid_len were P (the bucket): it does not
    // depend on valid_len, so its K/V are requested before that read returns.
    // With the suffix tiles first it is the true first tile unless the split
    // boundaries move; then the slot is drained and released (shift below).
    // Keys of the unit: the suffix tiles (none in prefill mode), then the
    // prefix rows [0, key limit).  The key limit is the valid length, or in
    // prefill mode the causal limit of this query block (no key past its last
    // query; nothing when the block lies wholly in the padding).
    const int TS = p.causal ? 0 : (p.S + NT - 1) / NT;
    auto key_limit = [&](int v) { return p.causal ? (q0 >= v ? 0 : min(v, q0 + nq)) : v; };
    const int t_bucket = TS + (key_limit(p.P) + NT - 1) / NT;
    const int g_spec = static_cast<int>((static_cast<long long>(t_bucket) * rank) / C);
    const bool spec =
        !p.prefix_static && g_spec < static_cast<int>((static_cast<long long>(t_bucket) * (rank + 1)) / C);
    uint64_t pol = 0;
    auto issue_q = [&]() {
        if (p.row_blocks == 1) {
            // both heads' S queries are contiguous: one 128-row box per chunk
            // (4-D view [units][rows][4 chunks][64]: one request lands all
            // four 64-column chunks, chunk-major, in the MMA layout)
            ptx::mbar_arrive_expect_tx(&bars[L::kBarQFull], L::kQBytes);
            ptx::tma_load_4d(sQ, &tm_q, &bars[L::kBarQFull], 0, 0, 0, unit);
        } else {
            // one SQ-row box per head and chunk, at 8-row-aligned rows h * rph
            ptx::mbar_arrive_expect_tx(&bars[L::kBarQFull], static_cast<uint32_t>(p.G * kChunks * p.SQ * 128));
            for (int h = 0; h < p.G; ++h)
                for (int c = 0; c < kChunks; ++c)
                    ptx::tma_load_3d(sQ + c * L::kQChunkBytes + h * rph * 128, &tm_q, &bars[L::kBarQFull],
                                     c * kChunkElems, h * p.S + q0, unit);
        }
    };
    if (warp == kProducerWarp && lane == 0) {
        pol = ptx::policy_evict_first();
        if (!p.prefix_static) issue_q();
        if (spec) {
            const TileInfo ti = tile_of<NT>(g_spec, TS, key_limit(p.P), p.S);
            const CUtensorMap *mk = ti.prefix ? &tm_kp : &tm_ks;
            const CUtensorMap *mv = ti.prefix ? &tm_vp : &tm_vs;
            ptx::mbar_arrive_expect_tx(&bars[L::kBarKFull], L::kTileBytes);
            ptx::tma_load_4d_hint(sK(0), mk, &bars[L::kBarKFull], 0, ti.row0, 0, unit, pol);
            ptx::mbar_arrive_expect_tx(&bars[L::kBarVFull], L::kTileBytes);
            ptx::tma_load_4d_hint(sV(0), mv, &bars[L::kBarVFull], 0, ti.row0, 0, unit, pol);
        }
    }

    int vl = p.P;
    if (p.valid_len != nullptr) {
        const int raw = __ldg(p.valid_len + b);
        vl = min(max(raw, 0), p.P);
        if (raw != vl && rank == 0 && threadIdx.x == 0) atomicOr(p.err, kEwClamped);
    }
    const int klim = key_limit(vl);
    // rows of the block that are written: every query, or in prefill mode
    // the queries before the valid length
    const int jlim = p.causal ? max(0, min(nq, vl - q0)) : nq;
    const int t_all = TS + (klim + NT - 1) / NT;
    const int t_begin = static_cast<int>((static_cast<long long>(t_all) * rank) / C);
    const int t_end = static_cast<int>((static_cast<long long>(t_all) * (rank + 1)) / C);
    const int T = t_end - t_begin;
    // K/V ring slot of tile t is t + shift: 0 when the early request was the
    // first tile, 1 when it was not (its slot is then skipped).
    const int shift = (spec && !(T > 0 && t_begin == g_spec)) ? 1 : 0;

    bool failed = false;

    if (warp == kProducerWarp) {
        // ================================================== TMA producer
        if (lane == 0) {
            int slots = spec ? 1 : 0;  // ring slots requested so far
            bool q_issued = !p.prefix_static;
            if (shift == 1) {
                // the early request is not one of this CTA's tiles: let it
                // land, then release its slot as its consumer would
                if (!ptx::mbar_wait(&bars[L::kBarKFull], 0, kWaitLimitNs) ||
                    !ptx::mbar_wait(&bars[L::kBarVFull], 0, kWaitLimitNs))
                    failed = true;
                ptx::mbar_arrive(&bars[L::kBarKEmpty]);
                ptx::mbar_arrive(&bars[L::kBarVEmpty]);
            }
            int k_issued = slots, v_issued = slots;
            for (int t = slots - shift; t < T && !failed; ++t) {
                const int slot = t + shift;
                const int s = slot % STAGES, n = slot / STAGES;
                const TileInfo ti = tile_of<NT>(t_begin + t, TS, klim, p.S);
                const CUtensorMap *mk = ti.prefix ? &tm_kp : &tm_ks;
                const CUtensorMap *mv = ti.prefix ? &tm_vp : &tm_vs;
                if (!q_issued && (!ti.prefix || slot >= STAGES - 1)) {
                    // Q and the suffix tensors may come from the preceding grid
                    ptx::griddep_wait();
                    issue_q();
                    q_issued = true;
                }
                if (n > 0 && !ptx::mbar_wait(&bars[L::kBarKEmpty + s], (n - 1) & 1, kWaitLimitNs)) {
                    failed = true;
                    break;
                }
                // the last stage first holds Q: wait until it is in TMEM
                if (slot == STAGES - 1 && !ptx::mbar_wait(&bars[L::kBarQFree], 0, kWaitLimitNs)) {
                    failed = true;
                    break;
                }
                ptx::mbar_arrive_expect_tx(&bars[L::kBarKFull + s], L::kTileBytes);
                ptx::tma_load_4d_hint(sK(s), mk, &bars[L::kBarKFull + s], 0, ti.row0, 0, unit, pol);
                DM05_TRACE_TILE(4, t);
                k_issued = slot + 1;
                if (n > 0 && !ptx::mbar_wait(&bars[L::kBarVEmpty + s], (n - 1) & 1, kWaitLimitNs)) {
                    failed = true;
                    break;
                }
                ptx::mbar_arrive_expect_tx(&bars[L::kBarVFull + s], L::kTileBytes);
                ptx::tma_load_4d_hint(sV(s), mv, &bars[L::kBarVFull + s], 0, ti.row0, 0, unit, pol);
                v_issued = slot + 1;
            }
            if (!q_issued) {
                ptx::griddep_wait();
                issue_q();
            }
            // Drain: every copy this thread issued must have landed before the
            // CTA may exit (normally all phases are long complete here).
            ptx::mbar_wait(&bars[L::kBarQFull], 0, kWaitLimitNs);
            for (int t = (k_issued > STAGES ? k_issued - STAGES : 0); t < k_issued; ++t)
                if (!ptx::mbar_wait(&bars[L::kBarKFull + t % STAGES], (t / STAGES) & 1, kWaitLimitNs)) failed = true;
            for (int t = (v_issued > STAGES ? v_issued - STAGES : 0); t < v_issued; ++t)
                if (!ptx::mbar_wait(&bars[L::kBarVFull + t % STAGES], (t / STAGES) & 1, kWaitLimitNs)) failed = true;
        }
    } else if (warp == kMmaWarp) {
        // ================================================== MMA issuer
        if (lane == 0 && T > 0) {
            constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(kMRows, kHeadDim, true);
            const uint32_t q_base = ptx::smem_addr(sQ);
            // operand descriptors of ring slot 0 (K-major K tile, MN-major V
            // tile); a slot or k-step offset is added to the start-address
            // field, which holds (address >> 4) in 14 bits (shared memory is
            // below 256 KB, so the sum never carries out of the field)
            const uint64_t kdesc0 = ptx::sw128_desc(ptx::smem_addr(sK(0)), 16, 1024);
            const uint64_t vdesc0 = ptx::sw128_desc(ptx::smem_addr(sV(0)), L::kTileChunkBytes, 1024);
            auto issue_pv = [&](int u) -> bool {
                const int s = (u + shift) % STAGES;
                const int pb = u % kSBufs;
                if (!ptx::mbar_wait(&bars[L::kBarPReady + pb], (u / kSBufs) & 1, kWaitLimitNs)) return false;
                if (!ptx::mbar_wait(&bars[L::kBarVFull + s], ((u + shift) / STAGES) & 1, kWaitLimitNs)) return false;
                DM05_TRACE_TILE(7, u);
                ptx::tc_fence_after_sync();
                // descriptor of V rows [0, 16) of this slot; each 16-row k-step
                // adds 16 * 128 bytes (in the 16-byte units of the address field)
                const uint64_t vdesc = vdesc0 + static_cast<uint64_t>((s * L::kStageBytes) >> 4);
                const uint32_t p_tmem = tmem + kTmemS + pb * NT;
                // only the 16-row k-steps that hold valid keys (a partial tile
                // stops early; the rows after its last valid key up to the
                // k-step end are zero)
                const int nk = (tile_of<NT>(t_begin + u, TS, klim, p.S).n_valid + 15) / 16;
#pragma unroll
                for (int kk = 0; kk < NT / 16; ++kk) {
                    if (kk >= nk) break;
                    // B = V rows [16kk, 16kk+16) of the tile, all 256 columns:
                    // 128-byte rows (16 B units), column chunks LBO apart,
                    // 8-row groups SBO apart.
                    ptx::mma_bf16_ts(tmem + kTmemO, p_tmem + kk * 8, vdesc + static_cast<uint64_t>((kk * 16 * 128) >> 4),
                                     idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
                }
                ptx::mma_commit(&bars[L::kBarVEmpty + s]);
                ptx::mma_commit(&bars[L::kBarPFree + pb]);
                DM05_TRACE_TILE(5, u);
                return true;
            };
            bool ok = ptx::mbar_wait(&bars[L::kBarQFull], 0, kWaitLimitNs);
            if (ok) {
                // Q -> TMEM once (row m to lane m, 16-column k-steps as 8
                // columns of bf16 pairs: the A layout of the QK MMAs below),
                // then the last ring stage is released to the producer.
                ptx::tc_fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk)
                    ptx::tmem_cp_128x256b(tmem + kTmemQ + kk * 8,
                                          ptx::sw128_desc(q_base + (kk >> 2) * L::kQChunkBytes + (kk & 3) * 32, 16, 1024));
                ptx::mma_commit(&bars[L::kBarQFree]);
                DM05_TRACE_CLOCK(3);
            }
            for (int t = 0; t < T && ok; ++t) {
                const int s = (t + shift) % STAGES;
                const int sb = t % kSBufs;
                if (!ptx::mbar_wait(&bars[L::kBarKFull + s], ((t + shift) / STAGES) & 1, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                if (t == 0) DM05_TRACE_CLOCK(14);
                DM05_TRACE_TILE(0, t);
                // S(t) overwrites the TMEM columns that held P(t - kSBufs): the
                // PV MMA reading them must have completed (issue order alone
                // does not order one MMA's operand reads before a later MMA's
                // accumulator writes).
                if (t >= kSBufs && !ptx::mbar_wait(&bars[L::kBarPFree + sb], (t / kSBufs - 1) & 1, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                DM05_TRACE_TILE(6, t);
                ptx::tc_fence_after_sync();
                const uint64_t kdesc = kdesc0 + static_cast<uint64_t>((s * L::kStageBytes) >> 4);
                const uint32_t d = tmem + kTmemS + sb * NT;
                // N = the whole tile (a compile-time instruction descriptor issues
                // faster than one built from the tile's valid keys); the softmax
                // masks every column past the valid ones, NaN rows included
                constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(kMRows, NT, false);
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk) {
                    // K-major, 128-byte swizzle: 16 elements = 32 bytes along
                    // the row; chunk kk/4 holds columns [64(kk/4), 64(kk/4)+64).
                    const uint32_t koff = ((kk >> 2) * L::kTileChunkBytes + (kk & 3) * 32) >> 4;
                    ptx::mma_bf16_ts(d, tmem + kTmemQ + kk * 8, kdesc + koff, idesc_qk, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(&bars[L::kBarKEmpty + s]);
                ptx::mma_commit(&bars[L::kBarSFull + sb]);
                DM05_TRACE_TILE(1, t);
                if (t > 0 && !issue_pv(t - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok) ok = issue_pv(T - 1);
            DM05_TRACE_CLOCK(4);
            // Wait for every MMA issued above before TMEM may be freed.
            ptx::mma_commit(&bars[L::kBarMmaFinal]);
            if (!ptx::mbar_wait(&bars[L::kBarMmaFinal], 0, kWaitLimitNs)) ok = false;
            DM05_TRACE_CLOCK(5);
            failed = !ok;
        }
    } else {
        // ================================================== softmax warps
        // Warp w owns TMEM lanes 32*(w%4).. (its 32 query rows) and half
        // hf = w/4 of every S tile's columns and of O's columns; the two
        // warps of a lane quarter exchange their row maxima and sums.
        const int q4 = warp & 3;
        const int hf = warp >> 2;
        const int row = q4 * 32 + lane;
        const int row_h = row / rph;
        const int row_j = row - row_h * rph;  // query of this row within its head's block
        const int tid = hf * 128 + row;  // 0..255 over the softmax threads
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        const uint8_t *mask_row = p.mask ? p.mask + static_cast<size_t>(b) * p.P : nullptr;
        float *xmax = reinterpret_cast<float *>(smem + L::kXchgOff);  // [2 tile parity][2 half][128 rows]
        float *xl = xmax + 2 * 2 * kMRows;                             // [2 half][128]
        float *xlh = xl + 2 * kMRows;                                  // [2 half][128]
        uint64_t *pair_bar = &bars[L::kBarPair + q4];
        int pair_phase = 0;
        auto pair_sync = [&]() -> bool {  // both warps of this lane quarter
            ptx::mbar_arrive(pair_bar);
            const bool ok = warp_wait(pair_bar, pair_phase & 1);
            ++pair_phase;
            return ok;
        };
        constexpr int NH = NT / 2;  // columns of a tile per half
        float m_used = -INFINITY;
        float l = 0.0f;   // this half's sum of fp32 probabilities (for the LSE)
        float lh = 0.0f;  // this half's sum of bf16-rounded probabilities (for O)
        // Prefix-mask bytes of this thread's columns of tile t (1 where no
        // mask applies), requested one tile ahead so that their latency hides
        // behind the previous tile instead of stalling the softmax.
        uint32_t mask_next[NH / 32];
        auto load_mask = [&](int t, uint32_t (&m)[NH / 32]) {
#pragma unroll
            for (int w = 0; w < NH / 32; ++w) m[w] = 1u;
            if (mask_row == nullptr || t >= T) return;
            const TileInfo tn = tile_of<NT>(t_begin + t, TS, klim, p.S);
            if (!tn.prefix) return;
#pragma unroll
            for (int w = 0; w < NH / 32; ++w) {
                const int c = hf * NH + w * 32 + lane;
                if (c < tn.n_valid) m[w] = __ldg(mask_row + tn.row0 + c);
            }
        };
        load_mask(0, mask_next);
        for (int t = 0; t < T; ++t) {
            const int sb = t % kSBufs;
            uint32_t mask_cur[NH / 32];
#pragma unroll
            for (int w = 0; w < NH / 32; ++w) mask_cur[w] = mask_next[w];
            load_mask(t + 1, mask_next);
            if (!warp_wait(&bars[L::kBarSFull + sb], (t / kSBufs) & 1)) {
                failed = true;
                break;
            }
            if (t == 0 && threadIdx.x == 0) DM05_TRACE_CLOCK(15);
            if (threadIdx.x == 0) DM05_TRACE_TILE(2, t);
            ptx::tc_fence_after_sync();
            const uint32_t scol = tmem + lane_base + kTmemS + sb * NT;
            uint32_t raw[NH / 16][16];
#pragma unroll
            for (int j = 0; j < NH / 16; ++j) ptx::tmem_ld16(scol + hf * NH + j * 16, raw[j]);
            ptx::tmem_ld_wait();

            const TileInfo ti = tile_of<NT>(t_begin + t, TS, klim, p.S);
            float s[NH];  // raw logits <q, k>; the scale is applied inside the exponent
#pragma unroll
            for (int c = 0; c < NH; ++c) s[c] = __uint_as_float(raw[c / 16][c % 16]);
            if (ti.n_valid < NT || (ti.prefix && mask_row != nullptr)) {
                // keys of this half that are out of range or hidden (the same
                // for every row) become -inf; a full tile without a mask has none
                uint32_t vis[NH / 32];
#pragma unroll
                for (int w = 0; w < NH / 32; ++w) {
                    const int c = hf * NH + w * 32 + lane;
                    const bool v = c < ti.n_valid && mask_cur[w] != 0u;
                    vis[w] = __ballot_sync(0xffffffffu, v);
                }
#pragma unroll
                for (int c = 0; c < NH; ++c)
                    if (!((vis[c / 32] >> (c % 32)) & 1u)) s[c] = -INFINITY;
            }
            if (p.causal && ti.row0 + NT - 1 > q0) {
                // prefill: key j is visible to query q0 + row_j only if j <= it
                const int over = ti.row0 + hf * NH - (q0 + row_j);  // key index - query index at c = 0
#pragma unroll
                for (int c = 0; c < NH; ++c)
                    if (c + over > 0) s[c] = -INFINITY;
            }
            // four independent chains, then combined (max is exact in any order)
            float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
            for (int c = 4; c < NH; ++c) m4[c % 4] = fmaxf(m4[c % 4], s[c]);
            float hmax = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            // log2 units; rounding is monotone, so this is the max of the scaled logits
            hmax *= p.scale_log2;
            // the row max over both halves
            xmax[((t & 1) * 2 + hf) * kMRows + row] = hmax;
            if (!pair_sync()) {
                failed = true;
                break;
            }
            const float tmax = fmaxf(hmax, xmax[((t & 1) * 2 + (hf ^ 1)) * kMRows + row]);
            // identical decision in both halves (same inputs)
            float factor = 1.0f;
            bool rescale_o = false;
            if (t == 0) {
                m_used = tmax;
            } else if (tmax > m_used + kRescaleThreshold) {
                factor = ptx::ex2(m_used - tmax);  // 0 when m_used is -inf
                rescale_o = true;
                l *= factor;
                lh *= factor;
                m_used = tmax;
            }
            const float msub = (m_used == -INFINITY) ? 0.0f : m_used;
            // p = 2^(s * scale - m) for a pair of columns at a time: the
            // exponent argument and both running sums use paired fp32 ops
            const uint64_t scale2 = ptx::f32x2(p.scale_log2, p.scale_log2);
            const uint64_t nm2 = ptx::f32x2(-msub, -msub);
            uint64_t l2 = ptx::f32x2(0.0f, 0.0f), lh2 = l2;
            uint32_t pk[NH / 2];
#pragma unroll
            for (int c = 0; c < NH; c += 2) {
                const float2 a = ptx::unpack_f32x2(ptx::fma_f32x2(ptx::f32x2(s[c], s[c + 1]), scale2, nm2));
                const float p0 = ptx::ex2(a.x), p1 = ptx::ex2(a.y);
                const uint32_t hb = pack_bf16x2(p0, p1);
                pk[c / 2] = hb;
                l2 = ptx::add_f32x2(l2, ptx::f32x2(p0, p1));
                lh2 = ptx::add_f32x2(lh2, ptx::f32x2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xffff0000u)));
            }
            const float2 lp = ptx::unpack_f32x2(l2), lhp = ptx::unpack_f32x2(lh2);
            l += lp.x + lp.y;
            lh += lhp.x + lhp.y;
#pragma unroll
            for (int j = 0; j < NH / 32; ++j) {
                uint32_t chunk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) chunk[e] = pk[j * 16 + e];
                ptx::tmem_st16(scol + hf * (NH / 2) + j * 16, chunk);
            }
            if (t > 0 && __any_sync(0xffffffffu, rescale_o)) {
                // O must hold the sum through PV(t-1), the last PV issued
                // (PV(t) waits for this warp's p_ready below): wait for its
                // completion on the free barrier of its S/P buffer.  The
                // parity is exact: PV(t-3), the previous use of that buffer,
                // completed before QK(t) could start, and PV(t+1) cannot
                // start before P(t+1) exists.
                if (!warp_wait(&bars[L::kBarPFree + (t - 1) % kSBufs], ((t - 1) / kSBufs) & 1)) {
                    failed = true;
                    break;
                }
                {
                    // this half's 128 columns of O (an all-zero O stays zero)
                    ptx::tc_fence_after_sync();
#pragma unroll 1
                    for (int j = 0; j < kHeadDim / 32; ++j) {
                        uint32_t o[16];
                        const uint32_t oc = tmem + lane_base + kTmemO + hf * (kHeadDim / 2) + j * 16;
                        ptx::tmem_ld16(oc, o);
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
                        ptx::tmem_st16(oc, o);
                    }
                }
            }
            ptx::tmem_st_wait();
            if (ti.prefix && (ti.n_valid & 15) != 0) {
                // Rows at or past valid_len may hold anything (NaN too) and
                // would poison O through 0 * NaN: clear the ones the last PV
                // k-step reads.
                const int st = (t + shift) % STAGES;
                if (!warp_wait(&bars[L::kBarVFull + st], ((t + shift) / STAGES) & 1)) {
                    failed = true;
                    break;
                }
                uint8_t *vt = sV(st);
                const int rows = (ti.n_valid + 15) / 16 * 16 - ti.n_valid;  // read by the last PV k-step
                const int units = kChunks * rows * 8;                       // 16-byte units
                for (int i = tid; i < units; i += kSoftmaxWarps * 32) {
                    const int c = i / (rows * 8);
                    const int rem = i - c * rows * 8;
                    const int r = ti.n_valid + rem / 8;
                    *reinterpret_cast<uint4 *>(vt + c * L::kTileChunkBytes + r * 128 + (rem & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                ptx::fence_proxy_async_smem();
            }
            ptx::tc_fence_before_sync();
            ptx::mbar_arrive(&bars[L::kBarPReady + sb]);
            if (threadIdx.x == 0) DM05_TRACE_TILE(3, t);
        }

        if (T == 0) {
            // Nothing to compute, but the early requests (Q, and the K/V of
            // the tile guessed before valid_len was known) still land in the
            // shared memory the split epilogue reuses: wait for them first.
            // (A CTA with tiles consumed them all before getting here.)
            if (!warp_wait(&bars[L::kBarQFull], 0)) failed = true;
            if (spec && (!warp_wait(&bars[L::kBarKFull], 0) || !warp_wait(&bars[L::kBarVFull], 0))) failed = true;
        }
        if (threadIdx.x == 0) DM05_TRACE_CLOCK(6);
        const bool have_o = T > 0 && !failed;
        if (have_o) {
            // the last PV (every earlier MMA completed before it)
            if (!warp_wait(&bars[L::kBarPFree + (T - 1) % kSBufs], ((T - 1) / kSBufs) & 1)) failed = true;
            ptx::tc_fence_after_sync();
        }
        if (threadIdx.x == 0) DM05_TRACE_CLOCK(7);
        // row sums over both halves
        xl[hf * kMRows + row] = l;
        xlh[hf * kMRows + row] = lh;
        if (!failed && !pair_sync()) failed = true;
        const float l_row = l + xl[(hf ^ 1) * kMRows + row];
        const float lh_row = lh + xlh[(hf ^ 1) * kMRows + row];
        const bool row_valid = row_h < p.G && row_j < jlim;
        const int row_k = row_h * nq + row_j;  // compact row (when valid)
        const size_t out_row = unit_row0 + static_cast<size_t>(row_h) * p.S + q0 + row_j;
        if (C == 1) {
            // ---------------------------------------- single CTA: normalise and store this half
            const float inv_l = 1.0f / lh_row;
#pragma unroll 1
            for (int j = 0; j < kHeadDim / 128; ++j) {
                uint32_t o[4][16];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                    ptx::tmem_ld16(tmem + lane_base + kTmemO + hf * (kHeadDim / 2) + j * 64 + qq * 16, o[qq]);
                ptx::tmem_ld_wait();
                if (row_valid) {
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(o[qq][2 * e]) * inv_l,
                                                                     __uint_as_float(o[qq][2 * e + 1]) * inv_l);
                            w[e] = *reinterpret_cast<uint32_t *>(&h);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(p.out + out_row * kHeadDim + hf * (kHeadDim / 2) +
                                                               j * 64 + qq * 16);
                        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            }
            if (hf == 0 && row_valid && p.lse != nullptr)
                p.lse[out_row] = (m_used + ptx::lg2(l_row)) * 0.69314718055994531f;
        } else {
            // ---------------------------------------- split: publish this CTA's partial
            // Row `row` of the partial: D fp32 of unnormalised O, then
            // {m, l, l_hat, 0}; each half stages its 128 columns, then one
            // bulk TMA store per row.
            const size_t prow = (static_cast<size_t>(cl) * C + rank) * (p.G * p.SQ) + row_k;
            uint8_t *srow = smem + row * L::kStageStride;
            const bool write_o = T > 0 && !failed;
            if (write_o) {
#pragma unroll 1
                for (int j = 0; j < kHeadDim / 128; ++j) {
                    uint32_t o[4][16];
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                        ptx::tmem_ld16(tmem + lane_base + kTmemO + hf * (kHeadDim / 2) + j * 64 + qq * 16, o[qq]);
                    ptx::tmem_ld_wait();
                    if (row_valid) {
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
                            uint4 *d = reinterpret_cast<uint4 *>(srow + (hf * (kHeadDim / 2) + j * 64 + qq * 16) * 4);
                            d[0] = make_uint4(o[qq][0], o[qq][1], o[qq][2], o[qq][3]);
                            d[1] = make_uint4(o[qq][4], o[qq][5], o[qq][6], o[qq][7]);
                            d[2] = make_uint4(o[qq][8], o[qq][9], o[qq][10], o[qq][11]);
                            d[3] = make_uint4(o[qq][12], o[qq][13], o[qq][14], o[qq][15]);
                        }
                    }
                }
            }
            if (row_valid) {
                if (hf == 0)
                    *reinterpret_cast<float4 *>(srow + kHeadDim * 4) =
                        make_float4(m_used, l_row, write_o ? lh_row : 0.0f, 0.0f);
                ptx::fence_proxy_async_smem();
            }
            // both halves of the row staged
            if (!failed && !pair_sync()) failed = true;
            if (threadIdx.x == 0) DM05_TRACE_TILE(3, 23);
            if (row_valid && hf == 0) {
                ptx::bulk_store_s2g(reinterpret_cast<uint8_t *>(p.part) + prow * L::kStageStride, ptx::smem_addr(srow),
                                    L::kStageStride);
                ptx::bulk_commit();
                ptx::bulk_wait_all();
                ptx::fence_proxy_async_global();
                if (threadIdx.x == 0) DM05_TRACE_CLOCK(8);
            }
        }
    }

    __syncwarp();
    if (C > 1) {
        // ================================================== split merge (rows)
        // Every CTA of the unit has published its partial; CTA `rank` now
        // combines rows [r_lo, r_hi) of all C partials:
        //   M = max_c m_c,  LH = sum_c lh_c 2^(m_c - M),  L = sum_c l_c 2^(m_c - M)
        //   out = sum_c 2^(m_c - M) O_c / LH,   lse = (M + log2 L) ln 2.
        if (threadIdx.x == 0) DM05_TRACE_CLOCK(9);
        ptx::cluster_sync();
        if (threadIdx.x == 0) DM05_TRACE_CLOCK(10);
        const int r_lo = (NR * rank) / C;  // compact rows of this query block
        const int r_hi = (NR * (rank + 1)) / C;
        const int nr = r_hi - r_lo;
        uint8_t *recv = smem;  // [C][nr] rows of kStageStride bytes
        // output row of each merged row (the softmax exchange area is free now;
        // nr <= NR <= 128 rows)
        long long *orow_s = reinterpret_cast<long long *>(smem + L::kXchgOff);
        if (nr > 0 && warp == 0) {
            if (lane == 0) ptx::mbar_arrive_expect_tx(&bars[L::kBarMerge], static_cast<uint32_t>(C * nr * L::kStageStride));
            __syncwarp();
            if (lane < C) {
                ptx::fence_proxy_async_global();
                ptx::bulk_load_g2s(ptx::smem_addr(smem) + static_cast<uint32_t>(lane * nr * L::kStageStride),
                                   reinterpret_cast<const uint8_t *>(p.part) +
                                       ((static_cast<size_t>(cl) * C + lane) * (p.G * p.SQ) + r_lo) * L::kStageStride,
                                   static_cast<uint32_t>(nr * L::kStageStride), &bars[L::kBarMerge]);
            }
        }
        if (nr > 0) {
            if (!warp_wait(&bars[L::kBarMerge], 0)) failed = true;
            if (threadIdx.x == 0) DM05_TRACE_CLOCK(11);
            // the host launches clusters of 2..kMaxSplits CTAs; any other
            // size is reported and merges nothing
            if (C <= kMaxSplits) {
                merge_weights<L>(recv, C, nr, p.lse, unit_row0, r_lo, nq, p.S, q0, jlim, orow_s);
                if (threadIdx.x == 0) DM05_TRACE_TILE(0, 23);
                __syncthreads();
                if (threadIdx.x == 0) DM05_TRACE_TILE(1, 23);
                merge_rows<L>(recv, C, nr, p.out, orow_s);
                if (threadIdx.x == 0) DM05_TRACE_TILE(2, 23);
            } else if (threadIdx.x == 0) {
                atomicOr(p.err, kEwBadSplit);
            }
        }
    }

    if (failed) atomicOr(p.err, kEwTimeout);
    if (threadIdx.x == 0) {
        DM05_TRACE_CLOCK(12);
        DM05_TRACE_GTIME(13);
    }
    __syncwarp();
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace dm05

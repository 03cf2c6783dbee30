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
//   * The two query heads of a GQA group form one MMA A operand:
//     M = G*S <= 128 rows (padded to 128 by TMA zero fill), K = D = 256.
//     Every K/V tile is therefore loaded once and used by both heads.
//   * Key rows are a list of 64-row tiles: the prefix rows [0, valid_len),
//     then the S suffix rows.  The CTAs of one unit split that list evenly
//     (the split depends on valid_len, read on the device, so a captured
//     graph stays valid for any valid_len).
//   * Warp roles: warp 4 issues TMA loads (Q once, then a ring of K and V
//     tiles); warp 5 allocates TMEM and issues tcgen05 MMAs from one thread;
//     warps 0-3 (one thread per query row = TMEM lane) run the softmax.
//   * S = Q K^T goes to TMEM (three rotating buffers).  The softmax thread of
//     row i reads its row with tcgen05.ld, applies the mask and the scale,
//     keeps a running max m and sum l, and writes P (bf16) back into the same
//     TMEM columns.  O += P V is a tcgen05 MMA with A = P read from TMEM and B
//     = the V tile in shared memory (MN-major).  O (128 x 256 fp32) lives in
//     TMEM for the whole pass.
//   * The running max is updated lazily: O and l are rescaled only when the
//     tile max exceeds the current max by more than 2^8 (exact: O and l use
//     the same stale max, and p <= 2^8 stays well inside fp32/bf16 range).
//   * Splits of one unit form a thread-block cluster.  At the end every CTA
//     scales its O by exp2(m_self - M) / L (M, L from the cluster's stats via
//     distributed shared memory), stages it in its own shared memory, and
//     each CTA sums one column slice over the cluster and writes bf16 output:
//     the split-KV merge happens on chip, with no workspace and no second
//     kernel.
//   * Every wait is bounded (2 s): on time-out the kernel records
//     DM05_EW_WAIT_TIMEOUT in the error word, drains its own copies and MMAs
//     (again bounded), frees TMEM and returns.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace dm05 {

constexpr int kHeadDim = 256;
constexpr int kMRows = 128;                       // MMA M: query rows (padded)
constexpr int kChunkElems = 64;                   // bf16 per 128-byte swizzle row
constexpr int kChunks = kHeadDim / kChunkElems;   // 4 column chunks of a row
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;                    // O: columns [0, 256)
constexpr uint32_t kTmemS = 256;                  // S/P buffers: [256, 256 + kSBufs*NT)
constexpr int kSBufs = 3;                         // S/P TMEM buffers in flight
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr float kRescaleThreshold = 8.0f;         // log2 units: p <= 2^8 between rescales
constexpr uint32_t kEwClamped = 0x1u;
constexpr uint32_t kEwTimeout = 0x2u;

struct KernelParams {
    const int32_t *valid_len;  // [B] or nullptr
    const uint8_t *mask;       // [B, P] or nullptr
    __nv_bfloat16 *out;        // [B*Hkv, GS, D]
    float *lse;                // [B*Hkv, GS] or nullptr
    uint32_t *err;             // device error word
    int Hkv, P, S, GS;         // GS = (Hq / Hkv) * S query rows of a unit
    int splits;                // CTAs per unit (cluster size)
    float scale_log2;          // log2(e) / sqrt(D)
};

template <int NT, int STAGES>
struct SmemLayout {
    static_assert(NT % 32 == 0 && NT >= 32 && kTmemS + kSBufs * NT <= kTmemCols, "tile rows");
    static constexpr int kQChunkBytes = kMRows * 128;                 // 16 KB
    static constexpr int kQBytes = kChunks * kQChunkBytes;            // 64 KB
    static constexpr int kTileChunkBytes = NT * 128;
    static constexpr int kTileBytes = kChunks * kTileChunkBytes;      // NT * 512
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQBytes;
    static constexpr int kVOff = kKOff + STAGES * kTileBytes;
    static constexpr int kDataEnd = kVOff + STAGES * kTileBytes;
    // barriers
    static constexpr int kBarQFull = 0;
    static constexpr int kBarKFull = 1;
    static constexpr int kBarKEmpty = kBarKFull + STAGES;
    static constexpr int kBarVFull = kBarKEmpty + STAGES;
    static constexpr int kBarVEmpty = kBarVFull + STAGES;
    static constexpr int kBarSFull = kBarVEmpty + STAGES;    // per S/P buffer
    static constexpr int kBarPReady = kBarSFull + kSBufs;    // per S/P buffer
    static constexpr int kBarPFree = kBarPReady + kSBufs;    // per S/P buffer
    static constexpr int kBarODone = kBarPFree + kSBufs;
    static constexpr int kBarMmaFinal = kBarODone + 1;
    static constexpr int kNumBars = kBarMmaFinal + 1;
    static constexpr int kBarOff = kDataEnd;
    static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
    static constexpr int kStatOff = (kTmemSlotOff + 16 + 15) / 16 * 16;  // m, l, l_hat [128] each
    static constexpr int kEnd = kStatOff + 3 * kMRows * 4;
    static constexpr int kAllocBytes = kEnd + 1024;                  // slack for 1 KB alignment
    // The cluster merge stages G*S rows x 1 KB of fp32 in the data region.
    static_assert(kDataEnd >= kMRows * kHeadDim * 4, "staging area must fit in the data region");
};

struct TileInfo {
    bool prefix;
    int row0;     // first key row (prefix row or suffix row index)
    int n_valid;  // rows of the tile that are in range
};

template <int NT>
__device__ __forceinline__ TileInfo tile_of(int g, int TP, int vl, int S)
{
    TileInfo ti;
    if (g < TP) {
        ti.prefix = true;
        ti.row0 = g * NT;
        ti.n_valid = min(NT, vl - ti.row0);
    } else {
        ti.prefix = false;
        ti.row0 = (g - TP) * NT;
        ti.n_valid = min(NT, S - ti.row0);
    }
    return ti;
}

// All lanes of a warp wait on the barrier; the result is made warp-uniform.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity)
{
    bool ok = ptx::mbar_wait(bar, parity, kWaitLimitNs);
    return __all_sync(0xffffffffu, ok);
}

// Packs two probabilities as bf16 (the MMA operand) and adds them to two
// running sums: the rounded values (which normalise O, so that O is an exact
// convex combination of V rows with the weights the MMA used) and the fp32
// values (which give the LSE).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi, float &sum_rounded, float &sum_exact)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    sum_rounded += __low2float(h) + __high2float(h);
    sum_exact += lo + hi;
    return *reinterpret_cast<uint32_t *>(&h);
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
    float *stat_m = reinterpret_cast<float *>(smem + L::kStatOff);
    float *stat_l = stat_m + kMRows;
    float *stat_lh = stat_l + kMRows;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int C = p.splits;
    const int unit = blockIdx.x / C;
    const int rank = blockIdx.x - unit * C;
    const int b = unit / p.Hkv;

    // ---- set-up that reads no input (overlaps the previous kernel under PDL)
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bars[L::kBarQFull], 1);
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
        ptx::mbar_init(&bars[L::kBarODone], 1);
        ptx::mbar_init(&bars[L::kBarMmaFinal], 1);
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

    // ---- from here on inputs are read: wait for the preceding grid
    ptx::griddep_wait();

    int vl = p.P;
    if (p.valid_len != nullptr) {
        const int raw = __ldg(p.valid_len + b);
        vl = min(max(raw, 0), p.P);
        if (raw != vl && rank == 0 && threadIdx.x == 0) atomicOr(p.err, kEwClamped);
    }
    const int TP = (vl + NT - 1) / NT;
    const int TS = (p.S + NT - 1) / NT;
    const int t_all = TP + TS;
    const int t_begin = static_cast<int>((static_cast<long long>(t_all) * rank) / C);
    const int t_end = static_cast<int>((static_cast<long long>(t_all) * (rank + 1)) / C);
    const int T = t_end - t_begin;

    uint8_t *sQ = smem + L::kQOff;
    uint8_t *sK = smem + L::kKOff;
    uint8_t *sV = smem + L::kVOff;
    bool failed = false;

    if (warp == kProducerWarp) {
        // ================================================== TMA producer
        if (lane == 0 && T > 0) {
            const uint64_t pol = ptx::policy_evict_first();
            ptx::mbar_arrive_expect_tx(&bars[L::kBarQFull], L::kQBytes);
            for (int c = 0; c < kChunks; ++c)
                ptx::tma_load_3d(sQ + c * L::kQChunkBytes, &tm_q, &bars[L::kBarQFull], c * kChunkElems, 0, unit);
            int k_issued = 0, v_issued = 0;
            for (int t = 0; t < T && !failed; ++t) {
                const int s = t % STAGES, n = t / STAGES;
                const TileInfo ti = tile_of<NT>(t_begin + t, TP, vl, p.S);
                const CUtensorMap *mk = ti.prefix ? &tm_kp : &tm_ks;
                const CUtensorMap *mv = ti.prefix ? &tm_vp : &tm_vs;
                if (n > 0 && !ptx::mbar_wait(&bars[L::kBarKEmpty + s], (n - 1) & 1, kWaitLimitNs)) {
                    failed = true;
                    break;
                }
                ptx::mbar_arrive_expect_tx(&bars[L::kBarKFull + s], L::kTileBytes);
                for (int c = 0; c < kChunks; ++c)
                    ptx::tma_load_3d_hint(sK + s * L::kTileBytes + c * L::kTileChunkBytes, mk, &bars[L::kBarKFull + s],
                                          c * kChunkElems, ti.row0, unit, pol);
                k_issued = t + 1;
                if (n > 0 && !ptx::mbar_wait(&bars[L::kBarVEmpty + s], (n - 1) & 1, kWaitLimitNs)) {
                    failed = true;
                    break;
                }
                ptx::mbar_arrive_expect_tx(&bars[L::kBarVFull + s], L::kTileBytes);
                for (int c = 0; c < kChunks; ++c)
                    ptx::tma_load_3d_hint(sV + s * L::kTileBytes + c * L::kTileChunkBytes, mv, &bars[L::kBarVFull + s],
                                          c * kChunkElems, ti.row0, unit, pol);
                v_issued = t + 1;
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
            constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(kMRows, NT, false);
            constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(kMRows, kHeadDim, true);
            const uint32_t q_base = ptx::smem_addr(sQ);
            const uint32_t k_base = ptx::smem_addr(sK);
            const uint32_t v_base = ptx::smem_addr(sV);
            auto issue_pv = [&](int u) -> bool {
                const int s = u % STAGES;
                const int pb = u % kSBufs;
                if (!ptx::mbar_wait(&bars[L::kBarPReady + pb], (u / kSBufs) & 1, kWaitLimitNs)) return false;
                if (!ptx::mbar_wait(&bars[L::kBarVFull + s], (u / STAGES) & 1, kWaitLimitNs)) return false;
                ptx::tc_fence_after_sync();
                const uint32_t vb = v_base + s * L::kTileBytes;
                const uint32_t p_tmem = tmem + kTmemS + pb * NT;
#pragma unroll
                for (int kk = 0; kk < NT / 16; ++kk) {
                    // B = V rows [16kk, 16kk+16) of the tile, all 256 columns:
                    // 128-byte rows (16 B units), column chunks LBO apart,
                    // 8-row groups SBO apart.
                    const uint64_t bdesc = ptx::sw128_desc(vb + kk * 16 * 128, L::kTileChunkBytes, 1024);
                    ptx::mma_bf16_ts(tmem + kTmemO, p_tmem + kk * 8, bdesc, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
                }
                ptx::mma_commit(&bars[L::kBarVEmpty + s]);
                ptx::mma_commit(&bars[L::kBarODone]);
                ptx::mma_commit(&bars[L::kBarPFree + pb]);
                return true;
            };
            bool ok = ptx::mbar_wait(&bars[L::kBarQFull], 0, kWaitLimitNs);
            for (int t = 0; t < T && ok; ++t) {
                const int s = t % STAGES;
                const int sb = t % kSBufs;
                if (!ptx::mbar_wait(&bars[L::kBarKFull + s], (t / STAGES) & 1, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                // S(t) overwrites the TMEM columns that held P(t - kSBufs): the
                // PV MMA reading them must have completed (issue order alone
                // does not order one MMA's operand reads before a later MMA's
                // accumulator writes).
                if (t >= kSBufs && !ptx::mbar_wait(&bars[L::kBarPFree + sb], (t / kSBufs - 1) & 1, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after_sync();
                const uint32_t kb = k_base + s * L::kTileBytes;
                const uint32_t d = tmem + kTmemS + sb * NT;
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk) {
                    // K-major, 128-byte swizzle: 16 elements = 32 bytes along
                    // the row; chunk kk/4 holds columns [64(kk/4), 64(kk/4)+64).
                    const uint32_t koff = (kk & 3) * 32;
                    const uint64_t adesc = ptx::sw128_desc(q_base + (kk >> 2) * L::kQChunkBytes + koff, 16, 1024);
                    const uint64_t bdesc = ptx::sw128_desc(kb + (kk >> 2) * L::kTileChunkBytes + koff, 16, 1024);
                    ptx::mma_bf16_ss(d, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(&bars[L::kBarKEmpty + s]);
                ptx::mma_commit(&bars[L::kBarSFull + sb]);
                if (t > 0 && !issue_pv(t - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok) ok = issue_pv(T - 1);
            // Wait for every MMA issued above before TMEM may be freed.
            ptx::mma_commit(&bars[L::kBarMmaFinal]);
            if (!ptx::mbar_wait(&bars[L::kBarMmaFinal], 0, kWaitLimitNs)) ok = false;
            failed = !ok;
        }
    } else {
        // ================================================== softmax warps
        const int row = warp * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint8_t *mask_row = p.mask ? p.mask + static_cast<size_t>(b) * p.P : nullptr;
        float m_used = -INFINITY;
        float l = 0.0f;   // sum of fp32 probabilities (for the LSE)
        float lh = 0.0f;  // sum of the bf16-rounded probabilities (for O)
        for (int t = 0; t < T; ++t) {
            const int sb = t % kSBufs;
            if (!warp_wait(&bars[L::kBarSFull + sb], (t / kSBufs) & 1)) {
                failed = true;
                break;
            }
            ptx::tc_fence_after_sync();
            const uint32_t scol = tmem + lane_base + kTmemS + sb * NT;
            uint32_t raw[NT / 16][16];
#pragma unroll
            for (int j = 0; j < NT / 16; ++j) ptx::tmem_ld16(scol + j * 16, raw[j]);
            ptx::tmem_ld_wait();

            const TileInfo ti = tile_of<NT>(t_begin + t, TP, vl, p.S);
            // visibility of the NT keys of this tile, same for every row
            uint32_t vis[NT / 32];
#pragma unroll
            for (int w = 0; w < NT / 32; ++w) {
                const int c = w * 32 + lane;
                bool v = c < ti.n_valid;
                if (v && ti.prefix && mask_row != nullptr) v = __ldg(mask_row + ti.row0 + c) != 0;
                vis[w] = __ballot_sync(0xffffffffu, v);
            }
            float s[NT];
            float tmax = -INFINITY;
#pragma unroll
            for (int c = 0; c < NT; ++c) {
                const float x = __uint_as_float(raw[c / 16][c % 16]) * p.scale_log2;
                s[c] = ((vis[c / 32] >> (c % 32)) & 1u) ? x : -INFINITY;
                tmax = fmaxf(tmax, s[c]);
            }
            float factor = 1.0f;
            bool rescale_o = false;
            if (t == 0) {
                m_used = tmax;
            } else if (tmax > m_used + kRescaleThreshold) {
                factor = ptx::ex2(m_used - tmax);  // 0 when m_used is -inf
                rescale_o = lh > 0.0f;             // otherwise O holds exact zeros
                l *= factor;
                lh *= factor;
                m_used = tmax;
            }
            const float msub = (m_used == -INFINITY) ? 0.0f : m_used;
            float lsum = 0.0f, lhsum = 0.0f;
            uint32_t pk[NT / 2];
#pragma unroll
            for (int c = 0; c < NT; c += 2)
                pk[c / 2] = pack_bf16x2(ptx::ex2(s[c] - msub), ptx::ex2(s[c + 1] - msub), lhsum, lsum);
            l += lsum;
            lh += lhsum;
#pragma unroll
            for (int j = 0; j < NT / 32; ++j) {
                uint32_t chunk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) chunk[e] = pk[j * 16 + e];
                ptx::tmem_st16(scol + j * 16, chunk);
            }
            if (t > 0) {
                // Every warp observes every PV completion in order (PV(t-1)
                // here), so the single o_done barrier is never two phases
                // ahead of a waiter and its parity is exact.  PV(t) cannot
                // start before this warp arrives on p_ready below.
                if (!warp_wait(&bars[L::kBarODone], (t - 1) & 1)) {
                    failed = true;
                    break;
                }
                if (__any_sync(0xffffffffu, rescale_o)) {
                    ptx::tc_fence_after_sync();
#pragma unroll 1
                    for (int j = 0; j < kHeadDim / 16; ++j) {
                        uint32_t o[16];
                        ptx::tmem_ld16(tmem + lane_base + kTmemO + j * 16, o);
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
                        ptx::tmem_st16(tmem + lane_base + kTmemO + j * 16, o);
                    }
                }
            }
            ptx::tmem_st_wait();
            if (ti.prefix && ti.n_valid < NT) {
                // Rows at or past valid_len may hold anything (NaN too) and
                // would poison O through 0 * NaN: clear them in the V tile.
                const int st = t % STAGES;
                if (!warp_wait(&bars[L::kBarVFull + st], (t / STAGES) & 1)) {
                    failed = true;
                    break;
                }
                uint8_t *vt = sV + st * L::kTileBytes;
                const int rows = NT - ti.n_valid;
                const int units = kChunks * rows * 8;  // 16-byte units
                for (int i = row; i < units; i += kSoftmaxWarps * 32) {
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
        }

        const bool have_o = T > 0 && !failed;
        if (have_o) {
            if (!warp_wait(&bars[L::kBarODone], (T - 1) & 1)) failed = true;
            ptx::tc_fence_after_sync();
        }
        const size_t out_row = static_cast<size_t>(unit) * p.GS + row;
        if (C == 1) {
            // ---------------------------------------- single CTA: normalise and store
            const float inv_l = 1.0f / lh;
#pragma unroll 1
            for (int j = 0; j < kHeadDim / 16; ++j) {
                uint32_t o[16];
                ptx::tmem_ld16(tmem + lane_base + kTmemO + j * 16, o);
                ptx::tmem_ld_wait();
                if (row < p.GS) {
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv_l,
                                                                 __uint_as_float(o[2 * e + 1]) * inv_l);
                        w[e] = *reinterpret_cast<uint32_t *>(&h);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(p.out + out_row * kHeadDim + j * 16);
                    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
            if (row < p.GS && p.lse != nullptr) p.lse[out_row] = (m_used + ptx::lg2(l)) * 0.69314718055994531f;
        } else {
            stat_m[row] = m_used;
            stat_l[row] = l;
            stat_lh[row] = lh;
        }
    }

    __syncwarp();
    if (C > 1) {
        // ================================================== on-chip split merge
        ptx::cluster_sync();  // stats of every CTA published
        float4 *stage = reinterpret_cast<float4 *>(smem);  // [128 rows][64 chunks], chunk index swizzled
        float lse_row = 0.0f;
        if (warp < kSoftmaxWarps) {
            const int row = warp * 32 + lane;
            const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
            const float m_self = stat_m[row], lh_self = stat_lh[row];
            float mr[16], lr[16], lhr[16];
            float M = -INFINITY;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                if (r < C) {
                    mr[r] = ptx::ld_dsmem_f32(ptx::mapa(ptx::smem_addr(&stat_m[row]), r));
                    lr[r] = ptx::ld_dsmem_f32(ptx::mapa(ptx::smem_addr(&stat_l[row]), r));
                    lhr[r] = ptx::ld_dsmem_f32(ptx::mapa(ptx::smem_addr(&stat_lh[row]), r));
                    M = fmaxf(M, mr[r]);
                }
            }
            float Lsum = 0.0f, LHsum = 0.0f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                if (r < C && lhr[r] > 0.0f) {
                    const float f = ptx::ex2(mr[r] - M);
                    Lsum += lr[r] * f;
                    LHsum += lhr[r] * f;
                }
            }
            const float wgt = (lh_self > 0.0f) ? ptx::ex2(m_self - M) / LHsum : 0.0f;
            lse_row = (M + ptx::lg2(Lsum)) * 0.69314718055994531f;
            ptx::fence_proxy_async_smem();
            const bool read_o = T > 0 && !failed && wgt != 0.0f;
#pragma unroll 1
            for (int j = 0; j < kHeadDim / 16; ++j) {
                uint32_t o[16];
                if (__any_sync(0xffffffffu, read_o)) {
                    ptx::tmem_ld16(tmem + lane_base + kTmemO + j * 16, o);
                    ptx::tmem_ld_wait();
                }
                if (row < p.GS) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int c = j * 4 + q4;
                        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (read_o) {
                            v.x = __uint_as_float(o[4 * q4 + 0]) * wgt;
                            v.y = __uint_as_float(o[4 * q4 + 1]) * wgt;
                            v.z = __uint_as_float(o[4 * q4 + 2]) * wgt;
                            v.w = __uint_as_float(o[4 * q4 + 3]) * wgt;
                        }
                        stage[row * 64 + (c ^ (row & 7))] = v;
                    }
                }
            }
        }
        ptx::cluster_sync();  // every CTA's scaled O staged
        {
            const int per = 64 / C;  // 16-byte column chunks owned by this CTA
            const int c_lo = rank * per;
            const int items = p.GS * per;
            const uint32_t stage_base = ptx::smem_addr(stage);
            for (int i = threadIdx.x; i < items; i += kThreads) {
                const int r = i / per;
                const int c = c_lo + (i - r * per);
                const uint32_t off = stage_base + static_cast<uint32_t>((r * 64 + (c ^ (r & 7))) * 16);
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int src = 0; src < C; ++src) {
                    const float4 v = ptx::ld_dsmem_f32x4(ptx::mapa(off, src));
                    acc.x += v.x;
                    acc.y += v.y;
                    acc.z += v.z;
                    acc.w += v.w;
                }
                __nv_bfloat162 h0 = __floats2bfloat162_rn(acc.x, acc.y);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(acc.z, acc.w);
                uint2 w2 = make_uint2(*reinterpret_cast<uint32_t *>(&h0), *reinterpret_cast<uint32_t *>(&h1));
                *reinterpret_cast<uint2 *>(p.out + (static_cast<size_t>(unit) * p.GS + r) * kHeadDim + c * 4) = w2;
            }
        }
        if (warp < kSoftmaxWarps && rank == 0 && p.lse != nullptr) {
            const int row = warp * 32 + lane;
            if (row < p.GS) p.lse[static_cast<size_t>(unit) * p.GS + row] = lse_row;
        }
        ptx::cluster_sync();  // no CTA leaves while a peer may still read its shared memory
    }

    if (failed) atomicOr(p.err, kEwTimeout);
    __syncwarp();
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace dm05

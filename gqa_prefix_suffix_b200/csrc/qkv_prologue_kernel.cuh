// qkv_prologue_kernel.cuh -- sm_100a kernel of the suffix attention's
// prologue: QKV projection, QK-Norm and RoPE in one pass.
//
// What it computes (page "TensorRT+Triton+FlexAttention: OpenDM VLA
// 快速推理加速栈深度剖析", section 2.2 lists "QKV projection + QK-Norm + RoPE
// done at once" among the fused steps; the action expert's shape table gives
// hidden 1024, head_dim 256, 8 / 4 heads): for token t (= b * S + i) and
// head hd of the weight's row order (Hq query heads, Hkv key heads, Hkv value
// heads),
//   y      = w[hd * D : (hd + 1) * D, :] x_t                    (projection)
//   y'     = y / sqrt(mean(y^2) + eps) * nw                     (query / key heads)
//   out_d  = y'_d cos(a_d) - y'_{d+D/2} sin(a_d),               d < D/2,
//   out_{d+D/2} = y'_d sin(a_d) + y'_{d+D/2} cos(a_d),  a_d = pos_t theta^(-2d/D)
// value heads are the plain projection.  Outputs go to q [B,Hq,S,D],
// k [B,Hkv,S,D], v [B,Hkv,S,D], the layout the suffix attention reads.
//
// Design (one CTA = MR feature rows of a head x one tile of NT tokens):
//   * Swapped GEMM on tcgen05: D^T[features, tokens] = W_rows x X^T with
//     M = MR feature rows (A, K-major from the weight; MR = 128, or 64 when
//     the grid is small, for twice the CTAs) and N = NT tokens (B, K-major
//     from the hidden states), K = H in 64-column chunks staged by TMA
//     (128-byte swizzle) in a ring.  The accumulator lives in TMEM.  The
//     64-row CTAs (one wave) stage four chunks at a time, so that every
//     weight and token row is read as 512 contiguous bytes.
//   * A CTA's MR feature rows are the two rotation partners of MR / 2 pairs:
//     features (MR/2) q + j (rows j) and (MR/2) q + 128 + j (rows MR/2 + j)
//     of its head, so RoPE needs no data from another CTA.  The 256 / MR CTAs
//     of a head form a cluster and exchange their per-token sums of squares
//     through distributed shared memory for the RMS norm.
//   * Epilogue: TMEM -> shared memory [MR][NT] fp32, per-token sums of
//     squares, the exchange, per-token 1 / rms and output row, then each
//     thread produces rotated pairs and stores bf16 (consecutive threads
//     write consecutive features).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace dm05 {
namespace prologue {

constexpr int kThreads = 128;
// Ring depth in 64-column K chunks: deep (about 192 KB, one CTA per SM)
// when the grid is about one wave and each CTA must keep its own weight
// stream's latency covered; shallow (about 96 KB, two CTAs per SM) when
// the grid spans several waves, so that one CTA's copies overlap the
// other's epilogue.
template <int NT, int MR = 128>
constexpr int deep_stages() { return (192 * 1024) / (MR * 128 + NT * 128) > 8 ? 8 : (192 * 1024) / (MR * 128 + NT * 128); }
template <int NT, int MR = 128>
constexpr int shallow_stages() { return (96 * 1024) / (MR * 128 + NT * 128); }
constexpr int kChunk = 64;                 // K columns per stage (128 bytes of bf16)
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kEwTimeout = 0x2u;

struct Params {
    const __nv_bfloat16 *qw;   // [D] query-norm weight
    const __nv_bfloat16 *kw;   // [D] key-norm weight
    const int32_t *pos;        // [T] positions
    __nv_bfloat16 *q, *k, *v;  // outputs
    uint32_t *err;
    int T, S, H, Hq, Hkv, D;   // tokens (B * S), tokens per sample, hidden, heads, head dim
    float eps;
    float log2_theta;          // log2(theta)
};

// MR feature rows per CTA (128, or 64 for small grids: twice the CTAs): the
// head's D features in 256 / MR CTAs of a cluster.
// W = K chunks per ring stage: 1, or 4 (one box of four chunks for each
// operand: every weight and token row read as 512 contiguous bytes)
template <int NT, int STAGES, int MR = 128, int W = 1>
struct Smem {
    static constexpr int kQ = 256 / MR;                  // CTAs (quarters or halves) per head
    static constexpr int kABytes = W * MR * kChunk * 2;  // MR feature rows of W K chunks
    static constexpr int kBBytes = W * NT * kChunk * 2;  // NT token rows
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = STAGES;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kYStride = NT + 1;              // fp32 per feature row (odd: conflict-free row writes)
    static constexpr int kYBytes = MR * kYStride * 4;
    // the epilogue tile and the per-group sums of squares reuse the ring
    static_assert(kRingBytes >= kYBytes + kThreads * 4 * 4, "the epilogue tile reuses the ring");
    static constexpr int kBarOff = kRingBytes;
    static constexpr int kNumBars = 2 * kStages + 1;     // full[s], empty[s], mma done
    static constexpr int kSsOff = kBarOff + kNumBars * 8 + 8;   // every CTA's sums of squares [kQ][NT]
    static constexpr int kInvOff = kSsOff + kQ * NT * 4;        // 1 / rms per token [NT]
    static constexpr int kPosOff = kInvOff + NT * 4;            // the tile's token positions [NT]
    static constexpr int kRowOff = (kPosOff + NT * 4 + 7) / 8 * 8;  // each token's output row offset [NT]
    static constexpr int kTmemSlotOff = kRowOff + NT * 8;
    static constexpr int kEnd = kTmemSlotOff + 16;
    static constexpr int kAllocBytes = kEnd + 1024;
};

// W = 4: tm_w is the 5-D view (64 columns, row, partner half -- row + 128 --,
// chunk of a 256-column group, group) with boxes of 64 x MR/2 x 2 x 4 x 1,
// and tm_x the 4-D view (64 columns, token, chunk, group) with boxes of
// 64 x NT x 4 x 1: each lands as four chunk-major [rows][128 B] blocks.
template <int NT, int STAGES, int MR, int W = 1>
__global__ void __launch_bounds__(kThreads, 1)
    qkv_prologue_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                        const Params p)
{
    static_assert(MR == 128 || MR == 64, "128 or 64 feature rows per CTA");
    static_assert(W == 1 || (W == 4 && MR == 64), "four K chunks per stage: the 64-row CTAs");
    using L = Smem<NT, STAGES, MR, W>;
    constexpr int kQ = L::kQ;
    constexpr int kHalf = MR / 2;  // rows per weight box: features [kHalf q, +kHalf) and [128 + kHalf q, +kHalf)
    static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "N of an M=128 MMA");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
    constexpr int kStages = L::kStages;
    uint64_t *full = bars, *empty = bars + kStages, *mma_done = bars + 2 * kStages;
    float *ss_all = reinterpret_cast<float *>(smem + L::kSsOff);  // [kQ][NT]: CTA r's sums at row r
    float *inv_s = reinterpret_cast<float *>(smem + L::kInvOff);
    int *pos_s = reinterpret_cast<int *>(smem + L::kPosOff);
    unsigned long long *row_s = reinterpret_cast<unsigned long long *>(smem + L::kRowOff);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kTmemSlotOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // blockIdx.x = (head * kQ + qi); blockIdx.y = token tile.  The kQ CTAs
    // of a head are one cluster.
    const int qi = blockIdx.x % kQ;
    const int hd = blockIdx.x / kQ;
    const int t0 = blockIdx.y * NT;
    const int D = p.D;
    const int n_chunks = p.H / kChunk / W;  // ring stages to stream (W = 4: the host checks H % 256)
    const bool is_v = hd >= p.Hq + p.Hkv;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        ptx::mbar_init(mma_done, 1);
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&tm_w);
        ptx::prefetch_tensormap(&tm_x);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, NT <= 32 ? 32 : NT <= 64 ? 64 : NT <= 128 ? 128 : 256);
        ptx::tmem_relinquish();
    }
    ptx::griddep_launch_dependents();
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    ptx::griddep_wait();
    // warps 2-3 (idle until the epilogue) fetch the tile's positions now, so
    // that the rotation loop below reads none from global memory
    for (int i = threadIdx.x - 64; i >= 0 && i < NT; i += kThreads - 64) pos_s[i] = t0 + i < p.T ? p.pos[t0 + i] : 0;

    bool failed = false;
    // feature rows of this CTA: the head's rows [kHalf*qi, +kHalf) then [kHalf*qi + 128, +kHalf)
    const int row_a = hd * D + kHalf * qi;
    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        for (int c = 0; c < n_chunks; ++c) {
            const int s = c % kStages, n = c / kStages;
            if (n > 0 && !ptx::mbar_wait(&empty[s], (n - 1) & 1, kWaitLimitNs)) {
                failed = true;
                break;
            }
            uint8_t *a = smem + s * L::kStageBytes;
            ptx::mbar_arrive_expect_tx(&full[s], L::kStageBytes);
            if constexpr (W == 4) {
                ptx::tma_load_5d(a, &tm_w, &full[s], 0, row_a, 0, 0, c);
                ptx::tma_load_4d(a + L::kABytes, &tm_x, &full[s], 0, t0, 0, c);
            } else {
                ptx::tma_load_2d(a, &tm_w, &full[s], c * kChunk, row_a);
                ptx::tma_load_2d(a + kHalf * 128, &tm_w, &full[s], c * kChunk, row_a + 128);
                ptx::tma_load_2d(a + L::kABytes, &tm_x, &full[s], c * kChunk, t0);
            }
        }
        // drain: every issued copy has landed before the CTA may exit
        for (int c = (n_chunks > kStages ? n_chunks - kStages : 0); c < n_chunks && !failed; ++c)
            if (!ptx::mbar_wait(&full[c % kStages], (c / kStages) & 1, kWaitLimitNs)) failed = true;
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = ptx::idesc_bf16_f32(MR, NT, false);
        const uint64_t adesc0 = ptx::sw128_desc(ptx::smem_addr(smem), 16, 1024);
        const uint64_t bdesc0 = ptx::sw128_desc(ptx::smem_addr(smem + L::kABytes), 16, 1024);
        bool ok = true;
        for (int c = 0; c < n_chunks; ++c) {
            const int s = c % kStages;
            if (!ptx::mbar_wait(&full[s], (c / kStages) & 1, kWaitLimitNs)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after_sync();
            const uint64_t so = static_cast<uint64_t>((s * L::kStageBytes) >> 4);
#pragma unroll
            for (int w = 0; w < W; ++w) {
                // chunk w of the stage: [MR rows][128 B] and [NT rows][128 B] blocks
                const uint64_t ao = so + static_cast<uint64_t>((w * MR * 128) >> 4);
                const uint64_t bo = so + static_cast<uint64_t>((w * NT * 128) >> 4);
#pragma unroll
                for (int kk = 0; kk < kChunk / 16; ++kk)
                    ptx::mma_bf16_ss(tmem, adesc0 + ao + static_cast<uint64_t>((kk * 32) >> 4),
                                     bdesc0 + bo + static_cast<uint64_t>((kk * 32) >> 4), idesc,
                                     (c > 0 || w > 0 || kk > 0) ? 1u : 0u);
            }
            ptx::mma_commit(&empty[s]);
        }
        ptx::mma_commit(mma_done);
        if (!ok) failed = true;
    }
    __syncwarp();

    // ---------------------------------------------------- epilogue
    // all MMAs (and so every stage's copies) complete
    if (!ptx::mbar_wait(mma_done, 0, kWaitLimitNs)) failed = true;
    ptx::tc_fence_after_sync();
    // columns = tokens; M = 128: TMEM lane = tile row; M = 64: tile row i sits
    // in lane 32 (i / 16) + i % 16 (lanes 0-15 of each warp's quarter)
    float *Y = reinterpret_cast<float *>(smem);  // [MR][kYStride]
    const int r = MR == 128 ? threadIdx.x : 16 * warp + lane;
    const bool holds_row = MR == 128 || lane < 16;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
    for (int j = 0; j < NT / 16; ++j) {
        uint32_t o[16];
        ptx::tmem_ld16(tmem + lane_base + j * 16, o);
        ptx::tmem_ld_wait();
        if (holds_row) {
#pragma unroll
            for (int e = 0; e < 16; ++e) Y[r * L::kYStride + j * 16 + e] = __uint_as_float(o[e]);
        }
    }
    __syncthreads();
    if (!is_v) {
        // per-token sum of squares over this CTA's MR features: thread
        // (token t, feature group g) sums MR / kGroups features with four
        // independent chains; the groups' sums meet in shared memory, and the
        // token's sum goes to every CTA of the head (row qi of ss_all)
        constexpr int kGroups = kThreads / NT > 0 ? kThreads / NT : 1;
        constexpr int kPer = MR / kGroups;
        static_assert(kPer % 4 == 0, "four chains");
        float *part = reinterpret_cast<float *>(smem + L::kYBytes);  // [kGroups][NT], after the tile
        for (int idx = threadIdx.x; idx < NT * kGroups; idx += kThreads) {
            const int t = idx % NT, g = idx / NT;
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            const float *col = Y + (g * kPer) * L::kYStride + t;
#pragma unroll 4
            for (int f = 0; f < kPer; f += 4) {
                const float y0 = col[(f + 0) * L::kYStride], y1 = col[(f + 1) * L::kYStride];
                const float y2 = col[(f + 2) * L::kYStride], y3 = col[(f + 3) * L::kYStride];
                a0 = fmaf(y0, y0, a0);
                a1 = fmaf(y1, y1, a1);
                a2 = fmaf(y2, y2, a2);
                a3 = fmaf(y3, y3, a3);
            }
            part[g * NT + t] = (a0 + a1) + (a2 + a3);
        }
        __syncthreads();
        for (int t = threadIdx.x; t < NT; t += kThreads) {
            float acc = 0.0f;
            for (int g = 0; g < kGroups; ++g) acc += part[g * NT + t];
            ss_all[qi * NT + t] = acc;
            const uint32_t a = ptx::smem_addr(ss_all + qi * NT + t);
#pragma unroll
            for (int rr = 1; rr < kQ; ++rr)
                ptx::st_dsmem_f32(ptx::mapa(a, static_cast<uint32_t>((qi + rr) % kQ)), acc);
        }
    }
    ptx::cluster_sync();  // every CTA's sums are in place (and no one still writes)

    // each thread: the two adjacent rotation pairs (fa, fa + D/2) and
    // (fa + 1, fa + 1 + D/2), fa = kHalf * qi + j0, for the tokens
    // t = tg (mod kGroupsT): bf16x2 stores, kTpt threads covering 4 kTpt
    // contiguous bytes per token and half
    constexpr int kTpt = kHalf / 2;              // threads per token
    constexpr int kGroupsT = kThreads / kTpt;    // token groups
    const int j0 = 2 * (threadIdx.x % kTpt);
    const int tg = threadIdx.x / kTpt;
    const int fa = kHalf * qi + j0;  // feature index within the head (first of the two pairs)
    const int fb = fa + D / 2;
    __nv_bfloat16 *dst_base;
    int heads, h;
    if (hd < p.Hq) {
        dst_base = p.q;
        heads = p.Hq;
        h = hd;
    } else if (!is_v) {
        dst_base = p.k;
        heads = p.Hkv;
        h = hd - p.Hq;
    } else {
        dst_base = p.v;
        heads = p.Hkv;
        h = hd - p.Hq - p.Hkv;
    }
    float wa0 = 1.0f, wa1 = 1.0f, wb0 = 1.0f, wb1 = 1.0f;
    double inv_freq0 = 0.0, inv_freq1 = 0.0;
    if (!is_v) {
        const __nv_bfloat16 *nw = hd < p.Hq ? p.qw : p.kw;
        wa0 = __bfloat162float(nw[fa]);
        wa1 = __bfloat162float(nw[fa + 1]);
        wb0 = __bfloat162float(nw[fb]);
        wb1 = __bfloat162float(nw[fb + 1]);
        // theta^(-2 f / D), in double: positions reach thousands of radians
        inv_freq0 = exp2(-2.0 * static_cast<double>(fa) / static_cast<double>(D) * static_cast<double>(p.log2_theta));
        inv_freq1 = exp2(-2.0 * static_cast<double>(fa + 1) / static_cast<double>(D) * static_cast<double>(p.log2_theta));
    }
    // Angle pos * inv_freq reduced to [-pi, pi] in fp32 without losing the
    // bits a large position carries: inv_freq is split into two floats, the
    // product's rounding error is recovered with an fma, and 2 pi is split
    // into three floats (Cody-Waite) with C1 = 6.28125 exact in few bits, so
    // that k * C1 and ph - k * C1 are exact for |k| < 2^16.  Worst error over
    // positions 0..4096 and all D / 2 frequencies (fp32 emulation against
    // fp64): 2.4e-7 rad.  Sine and cosine by the hardware approximation
    // (absolute error about 2^-21 on [-pi, pi]), far below the bf16 rounding.
    const float ih0 = static_cast<float>(inv_freq0), il0 = static_cast<float>(inv_freq0 - static_cast<double>(ih0));
    const float ih1 = static_cast<float>(inv_freq1), il1 = static_cast<float>(inv_freq1 - static_cast<double>(ih1));
    auto rot = [](float pos, float ih, float il, float &sn, float &cs) {
        const float ph = pos * ih;
        const float pe = fmaf(pos, ih, -ph) + pos * il;  // the product's rounding error, plus the low part
        const float k = rintf(ph * 0.159154943f);
        float r = fmaf(-k, 6.28125f, ph);                // exact
        r = fmaf(-k, 1.935307169e-03f, r);
        r = fmaf(-k, 1.025313168e-11f, r) + pe;
        __sincosf(r, &sn, &cs);
    };
    const int n_tok = min(NT, p.T - t0);
    // per token, once: 1 / rms (every CTA's sums arrived before the cluster
    // barrier), the position as a float, and the output row offset
    float *pos_f = reinterpret_cast<float *>(pos_s);
    if (threadIdx.x < n_tok) {
        const int t = threadIdx.x, tok = t0 + t;
        if (!is_v) {
            float tot = 0.0f;
            for (int rr = 0; rr < kQ; ++rr) tot += ss_all[rr * NT + t];  // the same order in every CTA
            inv_s[t] = rsqrtf(tot / static_cast<float>(D) + p.eps);
        }
        pos_f[t] = static_cast<float>(pos_s[t]);  // exact: positions are below 2^24
        const int bi = tok / p.S, i = tok - bi * p.S;
        row_s[t] = ((static_cast<unsigned long long>(bi) * heads + h) * p.S + i) * D;
    }
    __syncthreads();
#pragma unroll 4
    for (int t = tg; t < n_tok; t += kGroupsT) {
        const float ya0 = Y[j0 * L::kYStride + t], ya1 = Y[(j0 + 1) * L::kYStride + t];
        const float yb0 = Y[(kHalf + j0) * L::kYStride + t], yb1 = Y[(kHalf + 1 + j0) * L::kYStride + t];
        float oa0 = ya0, oa1 = ya1, ob0 = yb0, ob1 = yb1;
        if (!is_v) {
            const float inv_rms = inv_s[t];
            const float a0 = ya0 * inv_rms * wa0, a1 = ya1 * inv_rms * wa1;
            const float b0 = yb0 * inv_rms * wb0, b1 = yb1 * inv_rms * wb1;
            const float ps = pos_f[t];
            float sn0, cs0, sn1, cs1;
            rot(ps, ih0, il0, sn0, cs0);
            rot(ps, ih1, il1, sn1, cs1);
            oa0 = a0 * cs0 - b0 * sn0;
            ob0 = a0 * sn0 + b0 * cs0;
            oa1 = a1 * cs1 - b1 * sn1;
            ob1 = a1 * sn1 + b1 * cs1;
        }
        __nv_bfloat16 *row = dst_base + row_s[t];
        *reinterpret_cast<__nv_bfloat162 *>(row + fa) = __floats2bfloat162_rn(oa0, oa1);
        *reinterpret_cast<__nv_bfloat162 *>(row + fb) = __floats2bfloat162_rn(ob0, ob1);
    }

    if (failed && lane == 0) atomicOr(p.err, kEwTimeout);
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem, NT <= 32 ? 32 : NT <= 64 ? 64 : NT <= 128 ? 128 : 256);
    }
}

}  // namespace prologue
}  // namespace dm05

// post_attn_kernels.cuh -- sm_100a kernels of the post-attention block of an
// action-expert layer: output projection + residual, Adarms, GEGLU gate-up,
// MLP down + gated residual.
//
// What the block computes (page "TensorRT+Triton+FlexAttention: OpenDM VLA
// 快速推理加速栈深度剖析", section 2.2: after the three attention stages the
// suffix path chains the time modulation Adarms, the GEGLU gate-up and the MLP
// down; hidden 1024, intermediate 4096), for token t of sample b:
//   h1  = h_t + Wo a_t
//   u   = h1 / sqrt(mean(h1^2) + eps) * (1 + scale_b) + shift_b
//   m   = gelu_tanh(Wg u) * (Wu u)
//   out = h1 + gate_b * (Wd m)
//
// Design: the three projections are weight-streaming GEMMs with few tokens,
// so each is a swapped tcgen05 GEMM (gemm_kernel): D^T[weight rows, tokens]
// with M = 128 weight rows (A, K-major, 128-byte swizzle, TMA) and N = NT
// tokens (B, K-major), fp32 accumulation in TMEM, a TMA ring over 64-column
// K chunks.  A split-K grid dimension spreads a projection over more SMs; the
// fp32 partial tiles go to a workspace [split][token][row] and are summed in a
// fixed order by the row kernels that follow (deterministic, no atomics):
//   * Wo partials -> adarms_rows: residual, RMS norm over the hidden size,
//     time modulation; writes h1 (fp32) and u (bf16);
//   * Wgu (one CTA holds 64 gate rows and their 64 up rows) -> the GEGLU
//     epilogue inside the GEMM writes m (bf16);
//   * Wd partials -> gated_residual_rows: out = h1 + gate * sum (bf16).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace dm05 {
namespace post {

constexpr int kThreads = 128;
// ring depth: as many 64-column K chunks in flight as fit in ~192 KB (a CTA
// then has an SM to itself and keeps the weight stream's latency covered)
template <int NT>
constexpr int stages_for() { return (192 * 1024) / (128 * 128 + NT * 128) > 8 ? 8 : (192 * 1024) / (128 * 128 + NT * 128); }
constexpr int kChunk = 64;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kEwTimeout = 0x2u;

enum Epilogue : int {
    kPartial = 0,  // fp32 partial tile -> part[split][token][row]
    kGeglu = 1,    // rows: 64 gate + their 64 up rows -> m[token][f] = gelu_tanh(g) * up (bf16)
};

struct GemmParams {
    float *part;               // kPartial: [splits][T][N_rows] fp32
    __nv_bfloat16 *m;          // kGeglu: [T][F] bf16
    uint32_t *err;
    int T;                     // tokens (B * S)
    int S;                     // tokens per sample: a token tile never crosses samples
    int tiles_per_sample;      // ceil(S / NT)
    int xk_inner;              // K columns per row of the activation map's inner dimension
    int N_rows;                // rows of the weight (kPartial: output features)
    int F;                     // kGeglu: intermediate size (gate rows [0,F), up rows [F,2F))
    int chunks_per_split;      // K chunks each split covers
};

template <int NT>
struct GemmSmem {
    static constexpr int kABytes = 128 * kChunk * 2;
    static constexpr int kBBytes = NT * kChunk * 2;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = stages_for<NT>();
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kBarOff = kRingBytes;
    static constexpr int kNumBars = 2 * kStages + 1;
    static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8 + 8;
    static constexpr int kEnd = kTmemSlotOff + 16;
    static constexpr int kAllocBytes = kEnd + 1024;
};

__device__ __forceinline__ float gelu_tanh(float z)
{
    // z / 2 * (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3)))
    const float k0 = 0.7978845608028654f, k1 = 0.044715f;
    return 0.5f * z * (1.0f + tanhf(k0 * fmaf(k1 * z * z, z, z)));
}

// grid: x = row tile (128 weight rows), y = token tile (sample y / tiles,
// its tokens [NT * (y % tiles), +NT)), z = K split.  kPartial: the tile is
// weight rows [128 x, +128).  kGeglu: the tile is gate rows [64 x, +64)
// followed by up rows [F + 64 x, +64).  The activation map is 4-D
// [B][K / xk_inner][S][xk_inner]: K column k of token (b, i) sits at
// (k % xk_inner, i, k / xk_inner, b), which covers both a [B*S][K] matrix
// (xk_inner = K) and the attention output [B][Hq][S][D] read as the tokens'
// heads concatenated (xk_inner = D).
template <int NT, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                const GemmParams p)
{
    using L = GemmSmem<NT>;
    static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "N of an M=128 MMA");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
    constexpr int kStages = L::kStages;
    uint64_t *full = bars, *empty = bars + kStages, *mma_done = bars + 2 * kStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kTmemSlotOff);
    constexpr uint32_t kCols = NT <= 32 ? 32 : NT <= 64 ? 64 : NT <= 128 ? 128 : 256;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bs = blockIdx.y / p.tiles_per_sample;                 // sample
    const int i0 = (blockIdx.y - bs * p.tiles_per_sample) * NT;    // first token of the tile in the sample
    const int tok0 = bs * p.S + i0;                                // its token index
    const int n_tok = min(NT, p.S - i0);                           // valid tokens of the tile
    const int split = blockIdx.z;
    const int c_begin = split * p.chunks_per_split;
    const int n_chunks = p.chunks_per_split;
    const int row_a = EPI == kGeglu ? 64 * blockIdx.x : 128 * blockIdx.x;
    const int row_b = EPI == kGeglu ? p.F + 64 * blockIdx.x : row_a + 64;

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
        ptx::tmem_alloc(tmem_slot, kCols);
        ptx::tmem_relinquish();
    }
    ptx::griddep_launch_dependents();
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    ptx::griddep_wait();

    bool failed = false;
    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        for (int c = 0; c < n_chunks; ++c) {
            const int s = c % kStages, n = c / kStages;
            if (n > 0 && !ptx::mbar_wait(&empty[s], (n - 1) & 1, kWaitLimitNs)) {
                failed = true;
                break;
            }
            uint8_t *a = smem + s * L::kStageBytes;
            const int kc = (c_begin + c) * kChunk;
            ptx::mbar_arrive_expect_tx(&full[s], L::kStageBytes);
            ptx::tma_load_2d(a, &tm_w, &full[s], kc, row_a);
            ptx::tma_load_2d(a + 64 * 128, &tm_w, &full[s], kc, row_b);
            ptx::tma_load_4d(a + L::kABytes, &tm_x, &full[s], kc % p.xk_inner, i0, kc / p.xk_inner, bs);
        }
        for (int c = (n_chunks > kStages ? n_chunks - kStages : 0); c < n_chunks && !failed; ++c)
            if (!ptx::mbar_wait(&full[c % kStages], (c / kStages) & 1, kWaitLimitNs)) failed = true;
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, NT, false);
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
            for (int kk = 0; kk < kChunk / 16; ++kk)
                ptx::mma_bf16_ss(tmem, adesc0 + so + static_cast<uint64_t>((kk * 32) >> 4),
                                 bdesc0 + so + static_cast<uint64_t>((kk * 32) >> 4), idesc,
                                 (c > 0 || kk > 0) ? 1u : 0u);
            ptx::mma_commit(&empty[s]);
        }
        ptx::mma_commit(mma_done);
        if (!ok) failed = true;
    }
    __syncwarp();

    // ---------------------------------------------------- epilogue
    if (!ptx::mbar_wait(mma_done, 0, kWaitLimitNs)) failed = true;
    ptx::tc_fence_after_sync();
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    if (EPI == kPartial) {
        // thread = weight row (TMEM lane), its NT token values -> part[split][t][row]
        const int row = 128 * blockIdx.x + threadIdx.x;
        float *dst = p.part + (static_cast<size_t>(split) * p.T + tok0) * p.N_rows + row;
#pragma unroll
        for (int j = 0; j < NT / 16; ++j) {
            uint32_t o[16];
            ptx::tmem_ld16(tmem + lane_base + j * 16, o);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int jj = j * 16 + e;
                if (jj < n_tok) dst[static_cast<size_t>(jj) * p.N_rows] = __uint_as_float(o[e]);
            }
        }
    } else {
        // lanes 0-63: gate rows, lanes 64-127: the matching up rows; pass the
        // up values through shared memory (the ring is free now)
        float *up_s = reinterpret_cast<float *>(smem);  // [64][NT + 1]
        constexpr int kUS = NT + 1;
        if (warp >= 2) {
#pragma unroll
            for (int j = 0; j < NT / 16; ++j) {
                uint32_t o[16];
                ptx::tmem_ld16(tmem + lane_base + j * 16, o);
                ptx::tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) up_s[(threadIdx.x - 64) * kUS + j * 16 + e] = __uint_as_float(o[e]);
            }
        }
        __syncthreads();
        if (warp < 2) {
            const int f = 64 * blockIdx.x + threadIdx.x;
#pragma unroll
            for (int j = 0; j < NT / 16; ++j) {
                uint32_t o[16];
                ptx::tmem_ld16(tmem + lane_base + j * 16, o);
                ptx::tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int jj = j * 16 + e;
                    if (jj < n_tok) {
                        const float g = __uint_as_float(o[e]);
                        const float up = up_s[threadIdx.x * kUS + jj];
                        p.m[static_cast<size_t>(tok0 + jj) * p.F + f] = __float2bfloat16_rn(gelu_tanh(g) * up);
                    }
                }
            }
        }
    }

    if (failed && lane == 0) atomicOr(p.err, kEwTimeout);
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem, kCols);
    }
}

struct RowParams {
    const float *part;            // [splits][T][Hd] fp32 partial sums of a projection
    int splits;
    const __nv_bfloat16 *h;       // adarms: residual [T][Hd]
    const __nv_bfloat16 *scale;   // adarms: [B][Hd]
    const __nv_bfloat16 *shift;   // adarms: [B][Hd]
    const __nv_bfloat16 *gate;    // gated residual: [B][Hd]
    float *h1;                    // adarms writes, gated residual reads: [T][Hd] fp32
    __nv_bfloat16 *u;             // adarms: [T][Hd] bf16
    __nv_bfloat16 *out;           // gated residual: [T][Hd] bf16
    int T, S, Hd;
    float eps;
};

// One CTA per token: h1 = h + sum of the partials (fixed order), the RMS over
// Hd, then u = h1 / rms * (1 + scale) + shift.
__global__ void __launch_bounds__(256) adarms_rows(const RowParams p)
{
    __shared__ float red[8];
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const int t = blockIdx.x, b = t / p.S;
    float ss = 0.0f;
    for (int o = threadIdx.x; o < p.Hd; o += blockDim.x) {
        float acc = 0.0f;
        for (int sp = 0; sp < p.splits; ++sp) acc += p.part[(static_cast<size_t>(sp) * p.T + t) * p.Hd + o];
        const float x = __bfloat162float(p.h[static_cast<size_t>(t) * p.Hd + o]) + acc;
        p.h1[static_cast<size_t>(t) * p.Hd + o] = x;
        ss = fmaf(x, x, ss);
    }
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, k);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.0f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += red[w];
    const float inv_rms = rsqrtf(tot / static_cast<float>(p.Hd) + p.eps);
    for (int o = threadIdx.x; o < p.Hd; o += blockDim.x) {
        const float x = p.h1[static_cast<size_t>(t) * p.Hd + o];
        const float sc = __bfloat162float(p.scale[static_cast<size_t>(b) * p.Hd + o]);
        const float sh = __bfloat162float(p.shift[static_cast<size_t>(b) * p.Hd + o]);
        p.u[static_cast<size_t>(t) * p.Hd + o] = __float2bfloat16_rn(fmaf(x * inv_rms, 1.0f + sc, sh));
    }
}

// One CTA per token: out = h1 + gate * (sum of the partials).
__global__ void __launch_bounds__(256) gated_residual_rows(const RowParams p)
{
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const int t = blockIdx.x, b = t / p.S;
    for (int o = threadIdx.x; o < p.Hd; o += blockDim.x) {
        float acc = 0.0f;
        for (int sp = 0; sp < p.splits; ++sp) acc += p.part[(static_cast<size_t>(sp) * p.T + t) * p.Hd + o];
        const float g = __bfloat162float(p.gate[static_cast<size_t>(b) * p.Hd + o]);
        p.out[static_cast<size_t>(t) * p.Hd + o] = __float2bfloat16_rn(fmaf(g, acc, p.h1[static_cast<size_t>(t) * p.Hd + o]));
    }
}

}  // namespace post
}  // namespace dm05

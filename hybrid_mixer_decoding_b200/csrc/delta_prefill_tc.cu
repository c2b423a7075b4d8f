// Chunked delta-rule prefill in two passes, bf16 activations, fp32 state and accumulation,
// d_k = d_v = 128, chunk C = 64, on the 5th-generation tensor cores (tcgen05.mma into TMEM).
//
// Chunk algebra: the standard WY / UT-transform rewriting of the gated delta rule for the GDN and
// KDA mixers of "Super Apriel: One Checkpoint, Many Speeds" (abstract; gist.science technical
// summary, section 2a). For a chunk with start state M ([d_k][d_v] fp32) and G the per-channel
// cumulative log-gate inside the chunk (G_C its last row):
//   A_rs = beta_r sum_i k_ri k_si e^(G_ri - G_si)  (s < r),  P_rs = sum_i q_ri k_si e^(G_ri - G_si)
//   (s <= r),  T = (I + A)^-1 Diag(beta),  Kt = k e^G,  Qt = q e^G,  Kc = k e^(G_C - G)
//   W = T Kt,  Ut = T V,  U = Ut - W M,  O = Qt M + P U,  M_next = Diag(e^G_C) M + Kc^T U
// Everything up to W and Ut depends only on the chunk's own inputs; the last three lines carry
// the state from chunk to chunk.
//
// Pass A (prefill_prep_kernel): one CTA per (sequence, head, chunk), all chunks at once.
//  - q, k, v (and the KDA log-gates) arrive by 4-D TMA boxes in the 128-byte swizzled layout.
//  - Gate prefix in registers: thread (rg, cg) holds rows rg + 16 j (j < 4) of channels
//    8 cg .. 8 cg + 7; the 64-row prefix is four 16-lane shuffle scans (no CTA barrier).
//  - A and P: KDA as ONE M = 128 tcgen05.mma, [Kt; Qt] Kh^T with Kh = k e^-G, while every
//    cumulative log-gate of the chunk lies in [-80, 80] (the factors then stay inside fp32's
//    range); beyond that, A and P are formed directly from the exponent differences on the CUDA
//    cores, so no gate range is refused. GDN (scalar gate): [k; q] k^T on the tensor cores and
//    the decay e^(G_r - G_s) <= 1 applied per entry, which holds for any gate.
//  - T: the 16 x 16 diagonal blocks of (I + A)^-1 by row sweeps (fp32, one half-warp per
//    block, straight from the registers the A read-back left them in), then the blocks below
//    the diagonal on tf32 mma.sync, merging 16 -> 32 -> 64 (four dependent products):
//    X_ij = -X_ii sum_{k=j}^{i-1} A_ik X_kj.
//  - [W | Ut] = T [Kt | V] as M = 128 tcgen05.mma (token rows in TMEM lanes 0-63).
//  - One record per chunk: [-W; Qt], Kc, P, e^G_C, Ut (bf16 tiles in the operand layouts the
//    scan's tensor cores read; e^G_C fp32).
//  - The fused input activations are a template parameter, so the plain kernel carries none of
//    their code (a smaller kernel measured 2-3% faster).
// Pass B (prefill_scan_kernel): one CTA per (sequence, head, half of d_v) walks the chunks,
// warp-specialised: a producer warp streams records into a 3-stage ring with bulk copies (enough
// bytes in flight per SM to cover the copies' latency), one thread issues the tcgen05.mma
// products, eight warps hold the CTA's 64 fp32 state columns in registers (thread = row of d_k,
// 32 columns) and two warps drain the outputs. Per chunk (N = the CTA's 64 columns):
//   D_UO  = [-W; Qt] M                (M = 128, K = 128; lanes 0-63: -W M, 64-127: Qt M)
//   U     = Ut + (-W M)               (threads, bf16 operand)
//   D_UO += [- ; P] U,  D_S = Kc^T U  (lanes 64-127 of D_UO: O; D_S: the state increment)
//   M     = e^G_C M + D_S             (threads, fp32)
#include <cuda_runtime.h>

#include <algorithm>

#include "kernels.h"
#include "ptx.cuh"
#include "../../include/hmd.h"

namespace hmd {
namespace {

__device__ unsigned int g_err;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr float kLog2e = 1.4426950408889634f;
// Cumulative in-chunk log-gates in [-kPrefillFactorRange, kPrefillFactorRange] keep k e^G and
// k e^-G inside fp32's normal range, so A and P can be one tensor-core product (kernels.h).

// ---- the per-chunk record (bytes) ----------------------------------------------------------
constexpr uint32_t REC_WQ = 0;       // [-W; Qt] bf16, K-major: 2 halves of d_k x 128 rows x 128 B
constexpr uint32_t REC_KC = 32768;   // Kc [tok][d_k] bf16: 2 halves x 64 rows x 128 B
constexpr uint32_t REC_P = 49152;    // P [r][s] bf16: 64 rows x 128 B
constexpr uint32_t REC_GAM = 57344;  // e^{G_C} fp32 [128]
constexpr uint32_t REC_UT = 57856;   // Ut [tok][d_v] bf16: 2 halves x 64 rows x 128 B
constexpr uint32_t REC_BYTES = REC_UT + 16384;  // 74240
static_assert(REC_UT % 16 == 0 && REC_BYTES % 16 == 0, "bulk copies need 16-byte sizes");

// byte offset of bf16 element (row, col) of a tile whose 64-column halves hold `rows` rows,
// 128-byte XOR swizzle (the TMA / tensor-core layout)
__device__ __forceinline__ uint32_t toff(int row, int col, int rows) {
    return (uint32_t)((col >> 6) * rows * 128 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                      ((col & 7) << 1));
}
// byte offset of fp32 (row, ch), ch % 4 == 0, in the staged KDA log-gate tile: four 128-byte
// swizzled TMA boxes of [64 rows][32 channels]
__device__ __forceinline__ uint32_t goff(int r, int ch) {
    return (uint32_t)((ch >> 5) * 8192 + r * 128 + ((((ch & 31) >> 2) ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint8_t *record(const PrefillScanArgs &a, int bh, int c) {
    return static_cast<uint8_t *>(a.ws) + ((size_t)bh * a.n_seg + c) * REC_BYTES;
}

__device__ __forceinline__ float fexp(float x) { return ex2_approx(x * kLog2e); }

// fp32 scratch [64][64] in the Kt rows (0-63) of both 64-column halves of the [Kt; Qt] tile,
// which hold nothing before the factor pass: rows 0-31 in the first half, 32-63 in the second
__device__ __forceinline__ uint32_t atmp_off(int r, int s) {
    return (uint32_t)((r < 32 ? r * 256 : 16384 + (r - 32) * 256) + s * 4);
}

// ================================ pass A ==================================================
constexpr int kPrepThreads = 256;  // 8 warps, two CTAs per SM
constexpr uint32_t PA_KQ = 0;      // [Kt; Qt] bf16 K-major, 128 rows (q by TMA into rows 64-127;
                                   //   GDN: k also into rows 0-63); at the end [-W; Qt]
constexpr uint32_t PA_KH = 32768;  // k (TMA) -> Kh; after the A/P product: T bf16 [64][64]
                                   //   (rows 0-63 of the M = 128 operand) + warp scratch
constexpr uint32_t PA_V = 49152;   // v (TMA); after the W/Ut product: Ut (record layout)
constexpr uint32_t PA_G = 65536;   // KDA log-gates (TMA, fp32, 32 KB); then As, Xs fp32 [64][68]
constexpr uint32_t PA_AS = PA_G;
constexpr uint32_t PA_XS = PA_G + 17408;
constexpr uint32_t PA_SMALL = PA_G + 34816;  // 100352
constexpr uint32_t S_BETA = 0, S_NRM = 256, S_G = 768, S_BAR = 1024, S_TMEM = 1048,
                   S_SIZE = 1088;
constexpr uint32_t PA_SMEM = PA_SMALL + S_SIZE + 1024;
constexpr int AS_LD = 68;
constexpr int YS_LD = 24;
constexpr uint32_t PA_YS = PA_KH + 8192;  // four 16 x 24 fp32 tiles of the solve (rows 64-127
                                          // of the T operand: lanes the W/Ut read-back ignores)
constexpr uint32_t kPrepTmemCols = 256;
constexpr uint32_t ID_AP = idesc_bf16(128, 64, 0, 0);    // [Kt; Qt] Kh^T: both K-major
constexpr uint32_t ID_WU = idesc_bf16(128, 128, 0, 1);   // [T; -] [Kt | V]: B MN-major
static_assert(PA_YS + 4 * 16 * YS_LD * 4 <= PA_V, "warp scratch fits");
static_assert(PA_XS + 64 * AS_LD * 4 <= PA_SMALL, "solve tiles fit");

// acc += A B for 16 x 16 fp32 tiles in shared memory, on tf32 mma.sync m16n8k8 (g = lane / 4,
// t4 = lane % 4; acc[nt] is the accumulator fragment of columns 8 nt .. 8 nt + 7)
__device__ __forceinline__ void mma16_tf32(float (&acc)[2][4], const float *A, int lda,
                                           const float *Bm, int ldb, int g, int t4) {
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const float *ar = A + g * lda + 8 * ks + t4;
        const uint32_t af[4] = {to_tf32(ar[0]), to_tf32(ar[8 * lda]), to_tf32(ar[4]),
                                to_tf32(ar[8 * lda + 4])};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const float *br = Bm + (8 * ks + t4) * ldb + 8 * nt + g;
            mma_tf32_1688(acc[nt], af, to_tf32(br[0]), to_tf32(br[4 * ldb]));
        }
    }
}
// C = sgn * acc (fragment layout as above)
__device__ __forceinline__ void store16(float *C, int ldc, const float (&acc)[2][4], float sgn,
                                        int g, int t4) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int cc = 8 * nt + 2 * t4;
        C[g * ldc + cc] = sgn * acc[nt][0];
        C[g * ldc + cc + 1] = sgn * acc[nt][1];
        C[(g + 8) * ldc + cc] = sgn * acc[nt][2];
        C[(g + 8) * ldc + cc + 1] = sgn * acc[nt][3];
    }
}

// The 16 x 16 diagonal block bi of X = (I + A)^-1 by a row sweep in fp32, run by one half-warp:
// lane r (r = lane % 16) holds row r of the block, ar[s] = A_rs (s < r; the rest is ignored).
// After step s row s is final and every row below it subtracts A_rs times row s, which arrives
// by a shuffle. The row goes to Xs (fp32) and to T (bf16, times beta of its column).
__device__ __forceinline__ void diag_sweep(const float (&ar)[16], int bi, int r, float *Xs,
                                           uint8_t *Tt, const float *sbeta) {
    float x[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) x[c] = c == r ? 1.f : 0.f;
#pragma unroll
    for (int s = 0; s < 15; ++s) {
        const float f = r > s ? ar[s] : 0.f;
#pragma unroll
        for (int c = 0; c <= s; ++c) x[c] = fmaf(-f, __shfl_sync(0xffffffffu, x[c], s, 16), x[c]);
    }
    float *xr = Xs + (bi * 16 + r) * AS_LD + bi * 16;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
        *reinterpret_cast<float4 *>(xr + 4 * q4) = make_float4(x[4 * q4], x[4 * q4 + 1], x[4 * q4 + 2], x[4 * q4 + 3]);
    uint32_t w[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        w[e] = pack_bf16x2(x[2 * e] * sbeta[bi * 16 + 2 * e], x[2 * e + 1] * sbeta[bi * 16 + 2 * e + 1]);
    *reinterpret_cast<uint4 *>(Tt + toff(bi * 16 + r, bi * 16, 64)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4 *>(Tt + toff(bi * 16 + r, bi * 16 + 8, 64)) = make_uint4(w[4], w[5], w[6], w[7]);
}
// T's blocks above the diagonal are zero: 6 blocks x 16 rows x 32 B, by 128 threads (t < 128)
__device__ __forceinline__ void zero_upper_t(uint8_t *Tt, int t) {
    for (int idx = t; idx < 6 * 16 * 2; idx += 128) {
        const int blk = idx >> 5, rr = (idx >> 1) & 15, hh = idx & 1;
        const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);              // block row
        const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);  // block column > bi
        *reinterpret_cast<uint4 *>(Tt + toff(bi * 16 + rr, bj * 16 + hh * 8, 64)) = make_uint4(0, 0, 0, 0);
    }
}

template <bool KDA, bool FUSED>
__global__ void __launch_bounds__(kPrepThreads, 2)
prefill_prep_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmg,
                    const PrefillScanArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    float *As = reinterpret_cast<float *>(sm + PA_AS);
    float *Xs = reinterpret_cast<float *>(sm + PA_XS);
    float *sbeta = reinterpret_cast<float *>(sm + PA_SMALL + S_BETA);  // [64]
    float *nrm = reinterpret_cast<float *>(sm + PA_SMALL + S_NRM);     // [2][64] 1/|q|, 1/|k|
    float *sG = reinterpret_cast<float *>(sm + PA_SMALL + S_G);        // GDN: [64] prefix
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + PA_SMALL + S_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + PA_SMALL + S_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x / a.n_seg, c = blockIdx.x - bh * a.n_seg;
    const int b = bh / a.H, h = bh - b * a.H;
    const int T = a.T;
    const int t0 = (a.chunk_begin + c) * kC;
    const int n = min(kC, T - t0);
    uint8_t *rec = record(a, bh, c);
    const uint32_t bar_in = smem_u32(&bars[0]), bar_mma = smem_u32(&bars[1]),
                   bar_g = smem_u32(&bars[2]);
    constexpr bool fused = FUSED;  // raw projections (act.A_log set): activate them here

    if (tid == 0) {
        mbar_init(bar_in, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_g, 1);
        fence_barrier_init();
        prefetch_tmap(&tmq);
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        if constexpr (KDA) prefetch_tmap(&tmg);
    }
    griddep_launch_dependents();
    griddep_wait();  // the inputs may come from the previous kernel; the records' last reader is
                     // the previous scan
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), kPrepTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Abort after a wait gave up: let the copies and products in flight end (bounded), free the
    // tensor memory, report. Every thread of the CTA takes this path together.
    auto abort_cta = [&](uint32_t bar, uint32_t parity) {
        if (tid == 0) {
            atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
            (void)mbar_wait_bounded(bar, parity);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            __syncwarp();
            tc_fence_after();
            tmem_dealloc(tmem, kPrepTmemCols);
        }
    };

    // ---- inputs: q into the Qt rows, k into the Kh slot (GDN: also into the Kt rows), v, KDA
    //      log-gates, by TMA; rows past the end of the sequence read as zero ---------------------
    if (tid == 0) {
        if constexpr (KDA) {  // the log-gates first, on their own barrier: the gate pass needs
                              // nothing else
            mbar_arrive_expect_tx(bar_g, 4u * 8192u);
#pragma unroll
            for (int j = 0; j < 4; ++j) tma_load_4d(sb + PA_G + j * 8192, &tmg, bar_g, j * 32, h, t0, b);
        }
        mbar_arrive_expect_tx(bar_in, (KDA ? 6u : 8u) * 8192u);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(sb + PA_KQ + hf * 16384 + 8192, &tmq, bar_in, hf * 64, h, t0, b);
            tma_load_4d(sb + PA_KH + hf * 8192, &tmk, bar_in, hf * 64, h, t0, b);
            tma_load_4d(sb + PA_V + hf * 8192, &tmv, bar_in, hf * 64, h, t0, b);
            if constexpr (!KDA) tma_load_4d(sb + PA_KQ + hf * 16384, &tmk, bar_in, hf * 64, h, t0, b);
        }
        // the CTA that starts about one lifetime from now (one full wave of resident CTAs later)
        // finds its inputs in L2
        const int nx = (int)blockIdx.x + a.prefetch_stride;
        if (a.prefetch_stride > 0 && nx < (int)gridDim.x) {
            const int bh2 = nx / a.n_seg, c2 = nx - bh2 * a.n_seg;
            const int b2 = bh2 / a.H, h2 = bh2 - b2 * a.H, t2 = (a.chunk_begin + c2) * kC;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                tma_prefetch_4d(&tmq, hf * 64, h2, t2, b2);
                tma_prefetch_4d(&tmk, hf * 64, h2, t2, b2);
                tma_prefetch_4d(&tmv, hf * 64, h2, t2, b2);
            }
            if constexpr (KDA) {
#pragma unroll
                for (int j = 0; j < 4; ++j) tma_prefetch_4d(&tmg, j * 32, h2, t2, b2);
            }
        }
    }
    // thread (rg, cg): rows rg + 16 j, channels 8 cg .. 8 cg + 7 (the gate prefix and the factors)
    const int rg = tid & 15, cg = tid >> 4, ch0 = 8 * cg;
    float G[4][8];
    float Gtot[8];
    const float rate = fused ? expf(a.act.A_log[h]) : 0.f;
    if (tid < kC) {
        const size_t tok = ((size_t)b * T + t0 + tid) * a.H + h;
        float bt = tid < n ? a.beta[tok] : 0.f;
        if (fused && tid < n) bt = 1.f / (1.f + expf(-bt));
        sbeta[tid] = bt;
        if constexpr (!KDA) {  // GDN: inclusive prefix of the scalar log-gates over the chunk
            float x = tid < n ? a.log_gate[tok] : 0.f;
            if (fused && tid < n) x = -rate * hmd_softplus(x + a.act.dt_bias[h]);
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            sG[tid] = x;  // warp 1 adds warp 0's total below
        }
    }
    // KDA: the gate prefix in registers while q, k, v are still landing
    bool fallback = false;
    if constexpr (KDA) {
        if (__syncthreads_or(!mbar_wait_bounded(bar_g, 0))) {
            if (tid == 0) (void)mbar_wait_bounded(bar_in, 0);  // the other copies end first
            abort_cta(bar_g, 0);
            return;
        }
        const float *db = fused ? a.act.dt_bias + (size_t)h * kD + ch0 : nullptr;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = rg + 16 * j;
            const float4 x0 = *reinterpret_cast<const float4 *>(sm + PA_G + goff(r, ch0));
            const float4 x1 = *reinterpret_cast<const float4 *>(sm + PA_G + goff(r, ch0 + 4));
            G[j][0] = x0.x; G[j][1] = x0.y; G[j][2] = x0.z; G[j][3] = x0.w;
            G[j][4] = x1.x; G[j][5] = x1.y; G[j][6] = x1.z; G[j][7] = x1.w;
            if (fused) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    G[j][e] = r < n ? -rate * hmd_softplus(G[j][e] + db[e]) : 0.f;
            }
        }
        // inclusive prefix over the 64 rows: per quarter j a 16-lane scan over rg, plus the totals
        // of the quarters before it
#pragma unroll
        for (int e = 0; e < 8; ++e) Gtot[e] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float x = G[j][e];
#pragma unroll
                for (int off = 1; off < 16; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, off, 16);
                    if (rg >= off) x += y;
                }
                const float tot = __shfl_sync(0xffffffffu, x, 15, 16);
                G[j][e] = x + Gtot[e];
                Gtot[e] += tot;
            }
        }
        float mn = 0.f, mx = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                mn = fminf(mn, G[j][e]);
                mx = fmaxf(mx, G[j][e]);
            }
        }
        fallback = __syncthreads_or(mn < -kPrefillFactorRange || mx > kPrefillFactorRange);
        if (rg == 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                reinterpret_cast<float *>(rec + REC_GAM)[ch0 + e] = fexp(Gtot[e]);
        }
    }
    if (__syncthreads_or(!mbar_wait_bounded(bar_in, 0))) {
        abort_cta(bar_in, 0);
        return;
    }

    // ---- fused activations: 1/|q|, 1/|k| per row (4 threads per row, 32 channels each) ------
    if (fused) {
        const int r = tid >> 2, qq = tid & 3;
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            const int c0 = qq * 32 + c4 * 8;
            const uint4 qv = *reinterpret_cast<const uint4 *>(sm + PA_KQ + toff(64 + r, c0, 128));
            const uint4 kv = *reinterpret_cast<const uint4 *>(sm + PA_KH + toff(r, c0, 64));
            const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w}, kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sq += bf16_lo(qw[e]) * bf16_lo(qw[e]) + bf16_hi(qw[e]) * bf16_hi(qw[e]);
                sk += bf16_lo(kw[e]) * bf16_lo(kw[e]) + bf16_hi(kw[e]) * bf16_hi(kw[e]);
            }
        }
        sq += __shfl_xor_sync(0xffffffffu, sq, 1);
        sk += __shfl_xor_sync(0xffffffffu, sk, 1);
        sq += __shfl_xor_sync(0xffffffffu, sq, 2);
        sk += __shfl_xor_sync(0xffffffffu, sk, 2);
        if (qq == 0) {
            nrm[r] = rsqrtf(sq + a.act.eps);
            nrm[kC + r] = rsqrtf(sk + a.act.eps);
        }
    }
    if constexpr (!KDA) {
        if (tid >= 32 && tid < kC) sG[tid] += sG[31];  // complete the prefix (read before write:
                                                      //   warp 0's values are final)
    }
    __syncthreads();

    if constexpr (!KDA) {
        const float gc = sG[kC - 1];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int e = 0; e < 8; ++e) G[j][e] = sG[rg + 16 * j];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) Gtot[e] = gc;
        if (tid < kD) reinterpret_cast<float *>(rec + REC_GAM)[tid] = fexp(gc);
    }

    // ---- KDA beyond the factor range: A and P from the exponent differences themselves -------
    if constexpr (KDA) {
        if (fallback) {
            // G back into the gate tile (in place), then A (fp32 scratch in the Kt rows, free until
            // the factor pass) and P (bf16, record) by direct sums
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = rg + 16 * j;
                *reinterpret_cast<float4 *>(sm + PA_G + goff(r, ch0)) =
                    make_float4(G[j][0], G[j][1], G[j][2], G[j][3]);
                *reinterpret_cast<float4 *>(sm + PA_G + goff(r, ch0 + 4)) =
                    make_float4(G[j][4], G[j][5], G[j][6], G[j][7]);
            }
            __syncthreads();
            const int cgrp = tid & 7, rp = tid >> 3, c16 = 16 * cgrp;
#pragma unroll 1
            for (int pass = 0; pass < 2; ++pass) {
                const int r = pass == 0 ? rp : kC - 1 - rp;
                float gr[16], kr[16], qr[16];
                const float fq = fused ? nrm[r] : 1.f, fk = fused ? nrm[kC + r] : 1.f;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint4 kv = *reinterpret_cast<const uint4 *>(sm + PA_KH + toff(r, c16 + 8 * u, 64));
                    const uint4 qv = *reinterpret_cast<const uint4 *>(sm + PA_KQ + toff(64 + r, c16 + 8 * u, 128));
                    const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w}, qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        kr[8 * u + 2 * e] = fk * bf16_lo(kw[e]);
                        kr[8 * u + 2 * e + 1] = fk * bf16_hi(kw[e]);
                        qr[8 * u + 2 * e] = fq * bf16_lo(qw[e]);
                        qr[8 * u + 2 * e + 1] = fq * bf16_hi(qw[e]);
                    }
#pragma unroll
                    for (int e4 = 0; e4 < 2; ++e4) {
                        const float4 g4 = *reinterpret_cast<const float4 *>(sm + PA_G + goff(r, c16 + 8 * u + 4 * e4));
                        gr[8 * u + 4 * e4] = g4.x; gr[8 * u + 4 * e4 + 1] = g4.y;
                        gr[8 * u + 4 * e4 + 2] = g4.z; gr[8 * u + 4 * e4 + 3] = g4.w;
                    }
                }
                const float br = r < n ? sbeta[r] : 0.f;
#pragma unroll 1
                for (int s = 0; s <= r; ++s) {
                    float aa = 0.f, pp = 0.f;
                    const float fks = fused ? nrm[kC + s] : 1.f;
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const uint4 kv = *reinterpret_cast<const uint4 *>(sm + PA_KH + toff(s, c16 + 8 * u, 64));
                        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                        for (int e4 = 0; e4 < 2; ++e4) {
                            const float4 g4 = *reinterpret_cast<const float4 *>(sm + PA_G + goff(s, c16 + 8 * u + 4 * e4));
                            const float gs[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int ci = 8 * u + 4 * e4 + e;
                                const uint32_t w = kw[(4 * e4 + e) >> 1];
                                const float ks = fks * (((4 * e4 + e) & 1) ? bf16_hi(w) : bf16_lo(w));
                                const float d = fexp(gr[ci] - gs[e]) * ks;
                                aa += kr[ci] * d;
                                pp += qr[ci] * d;
                            }
                        }
                    }
#pragma unroll
                    for (int m = 1; m < 8; m <<= 1) {
                        aa += __shfl_xor_sync(0xffffffffu, aa, m);
                        pp += __shfl_xor_sync(0xffffffffu, pp, m);
                    }
                    if (cgrp == 0) {
                        *reinterpret_cast<float *>(sm + PA_KQ + atmp_off(r, s)) = s < r ? br * aa : 0.f;
                        *reinterpret_cast<__nv_bfloat16 *>(rec + REC_P + toff(r, s, 64)) =
                            __float2bfloat16_rn(r < n ? pp : 0.f);
                    }
                }
                if (cgrp == 0) {  // the rest of the row of P is zero
                    for (int s = r + 1; s < kC; ++s)
                        *reinterpret_cast<__nv_bfloat16 *>(rec + REC_P + toff(r, s, 64)) =
                            __float2bfloat16_rn(0.f);
                }
            }
            __syncthreads();
            // A -> As (ld 68), zero on and above the diagonal; the gate tile is dead now
            for (int idx = tid; idx < kC * kC; idx += kPrepThreads) {
                const int r = idx >> 6, s = idx & 63;
                As[r * AS_LD + s] = s < r ? *reinterpret_cast<const float *>(sm + PA_KQ + atmp_off(r, s)) : 0.f;
            }
            __syncthreads();
        }
    }

    // ---- factors: Kt, Qt (and KDA's Kh) into shared memory, Kc into the record --------------
    {
        float gce[8];  // e^G_C of this thread's channels
#pragma unroll
        for (int e = 0; e < 8; ++e) gce[e] = fexp(Gtot[e]);
        float fq[4], fk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            fq[j] = fused ? nrm[rg + 16 * j] : 1.f;
            fk[j] = fused ? nrm[kC + rg + 16 * j] : 1.f;
        }
        if constexpr (!KDA) {
            // GDN: the A/P product reads raw [k; q] and k first; it runs while Kc is formed, and
            // Kt, Qt overwrite [k; q] once it is done
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t ad = smem_desc_sw128(sb + PA_KQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(sb + PA_KH + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                    umma_bf16(tmem, ad, bd, ID_AP, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar_mma);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = rg + 16 * j;
            const uint4 kv = *reinterpret_cast<const uint4 *>(sm + PA_KH + toff(r, ch0, 64));
            const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
            uint32_t kcw[4];
            if constexpr (KDA) {
                const uint4 qv = *reinterpret_cast<const uint4 *>(sm + PA_KQ + toff(64 + r, ch0, 128));
                const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
                uint32_t kt[4], qt[4], kh[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float ga = G[j][2 * e], gb = G[j][2 * e + 1];
                    const float ea = fexp(ga), eb = fexp(gb);
                    const float ia = fexp(-ga), ib = fexp(-gb);
                    const float ka = fk[j] * bf16_lo(kw[e]), kb = fk[j] * bf16_hi(kw[e]);
                    const float qa = fq[j] * bf16_lo(qw[e]), qb = fq[j] * bf16_hi(qw[e]);
                    kt[e] = pack_bf16x2(ka * ea, kb * eb);
                    qt[e] = pack_bf16x2(qa * ea, qb * eb);
                    kh[e] = pack_bf16x2(ka * ia, kb * ib);
                    // e^(G_C - G) <= 1: from e^-G while that is finite, else directly
                    kcw[e] = fallback ? pack_bf16x2(ka * fexp(Gtot[2 * e] - ga), kb * fexp(Gtot[2 * e + 1] - gb))
                                      : pack_bf16x2(ka * (gce[2 * e] * ia), kb * (gce[2 * e + 1] * ib));
                }
                *reinterpret_cast<uint4 *>(sm + PA_KQ + toff(r, ch0, 128)) = make_uint4(kt[0], kt[1], kt[2], kt[3]);
                *reinterpret_cast<uint4 *>(sm + PA_KQ + toff(64 + r, ch0, 128)) =
                    make_uint4(qt[0], qt[1], qt[2], qt[3]);
                if (!fallback)
                    *reinterpret_cast<uint4 *>(sm + PA_KH + toff(r, ch0, 64)) =
                        make_uint4(kh[0], kh[1], kh[2], kh[3]);
            } else {
                const float ec = fexp(Gtot[0] - G[j][0]) * fk[j];
#pragma unroll
                for (int e = 0; e < 4; ++e) kcw[e] = pack_bf16x2(ec * bf16_lo(kw[e]), ec * bf16_hi(kw[e]));
            }
            *reinterpret_cast<uint4 *>(rec + REC_KC + toff(r, ch0, 64)) =
                make_uint4(kcw[0], kcw[1], kcw[2], kcw[3]);
        }
    }
    if constexpr (KDA) {
        fence_proxy_async_smem();  // Kt, Qt, Kh are read by the tensor cores
        __syncthreads();
        if (!fallback && tid == 0) {  // [A_raw; P] = [Kt; Qt] Kh^T into TMEM columns 0-63
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
                const uint64_t ad = smem_desc_sw128(sb + PA_KQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(sb + PA_KH + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                umma_bf16(tmem, ad, bd, ID_AP, kk > 0 ? 1u : 0u);
            }
            umma_commit(bar_mma);
        }
    }

    // ---- A (fp32, masked, times beta) and P (bf16, record) from the product ------------------
    if (!fallback) {
        if (__syncthreads_or(!mbar_wait_bounded(bar_mma, 0))) {
            abort_cta(bar_mma, 0);
            return;
        }
        tc_fence_after();
        // warp w reads TMEM lanes 32 (w & 3) .. +31 (one row each), columns 32 (w >> 2) .. +31
        const int quad = warp & 3, s0 = 32 * (warp >> 2);
        uint32_t d[32];
        tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + s0, d);
        tmem_wait_ld();
        const int r = 32 * (quad & 1) + lane;
        float dec[32];  // GDN: e^(G_r - G_s) and the norms; KDA: 1
#pragma unroll
        for (int e = 0; e < 32; ++e) dec[e] = 1.f;
        if constexpr (!KDA) {
            const float gr = sG[r];
            const float fr = fused ? nrm[(quad < 2 ? kC : 0) + r] : 1.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int s = s0 + e;
                dec[e] = (s <= r ? fexp(gr - sG[s]) : 0.f) * fr * (fused ? nrm[kC + s] : 1.f);
            }
        }
        if (quad < 2) {  // A_rs = beta_r (.)_rs, s < r
            const float br = r < n ? sbeta[r] : 0.f;
            float *arow = As + r * AS_LD + s0;
            float av[32];
#pragma unroll
            for (int ee = 0; ee < 32; ++ee) av[ee] = (s0 + ee < r) ? br * dec[ee] * __uint_as_float(d[ee]) : 0.f;
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4)
                *reinterpret_cast<float4 *>(arow + 4 * j4) =
                    make_float4(av[4 * j4], av[4 * j4 + 1], av[4 * j4 + 2], av[4 * j4 + 3]);
            // warp 0 (rows 0-31, columns 0-31) holds diagonal blocks 0 and 1, warp 5 (rows 32-63,
            // columns 32-63) blocks 2 and 3, one per half-warp: sweep them from these registers
            if (warp == 0 || warp == 5) {
                const int hh = lane >> 4;
                float ar[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) ar[e] = hh ? av[16 + e] : av[e];
                diag_sweep(ar, 2 * (warp == 5) + hh, lane & 15, Xs, sm + PA_KH, sbeta);
            }
        } else {  // P_rs, s <= r
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int ee = 8 * u + 2 * e, s = s0 + ee;
                    w[e] = pack_bf16x2((s <= r && r < n) ? dec[ee] * __uint_as_float(d[ee]) : 0.f,
                                       (s + 1 <= r && r < n) ? dec[ee + 1] * __uint_as_float(d[ee + 1]) : 0.f);
                }
                *reinterpret_cast<uint4 *>(rec + REC_P + toff(r, s0 + 8 * u, 64)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
            zero_upper_t(sm + PA_KH, (warp >> 2) * 64 + (quad - 2) * 32 + lane);
        }
        tc_fence_before();
        __syncthreads();
    }
    if constexpr (!KDA) {
        // GDN: Kt, Qt over [k; q] now that the product has read them
        float fq[4], fk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            fq[j] = fused ? nrm[rg + 16 * j] : 1.f;
            fk[j] = fused ? nrm[kC + rg + 16 * j] : 1.f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = rg + 16 * j;
            const float eg = fexp(G[j][0]);
            const uint4 kv = *reinterpret_cast<const uint4 *>(sm + PA_KQ + toff(r, ch0, 128));
            const uint4 qv = *reinterpret_cast<const uint4 *>(sm + PA_KQ + toff(64 + r, ch0, 128));
            const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w}, qw[4] = {qv.x, qv.y, qv.z, qv.w};
            uint32_t kt[4], qt[4];
            const float sk = eg * fk[j], sq = eg * fq[j];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                kt[e] = pack_bf16x2(sk * bf16_lo(kw[e]), sk * bf16_hi(kw[e]));
                qt[e] = pack_bf16x2(sq * bf16_lo(qw[e]), sq * bf16_hi(qw[e]));
            }
            *reinterpret_cast<uint4 *>(sm + PA_KQ + toff(r, ch0, 128)) = make_uint4(kt[0], kt[1], kt[2], kt[3]);
            *reinterpret_cast<uint4 *>(sm + PA_KQ + toff(64 + r, ch0, 128)) = make_uint4(qt[0], qt[1], qt[2], qt[3]);
        }
    }

    // ---- T = (I + A)^-1 Diag(beta) ---------------------------------------------------------
    uint8_t *Tt = sm + PA_KH;  // bf16 [r][s], K-major, rows 0-63 of the W/Ut product's A operand
    // the diagonal blocks: swept from the read-back registers above, or here after the
    // CUDA-core A of a chunk beyond the factor range (then from As)
    if (fallback) {
        if (warp < 2) {
            const int bi = 2 * warp + (lane >> 4), r = lane & 15;
            const float *ap = As + (bi * 16 + r) * AS_LD + bi * 16;
            float ar[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 v = *reinterpret_cast<const float4 *>(ap + 4 * q4);
                ar[4 * q4] = v.x; ar[4 * q4 + 1] = v.y; ar[4 * q4 + 2] = v.z; ar[4 * q4 + 3] = v.w;
            }
            diag_sweep(ar, bi, r, Xs, Tt, sbeta);
        } else if (warp >= 4) {
            zero_upper_t(Tt, tid - 128);
        }
        __syncthreads();
    }
    {
        const int g8 = lane >> 2, t4 = lane & 3;
        float *Ys = reinterpret_cast<float *>(sm + PA_YS);
        auto store_t = [&](int bi, int bj, const float (&acc)[2][4], float sgn) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int cc = 16 * bj + 8 * nt + 2 * t4;
                const float b0 = sgn * sbeta[cc], b1 = sgn * sbeta[cc + 1];
                *reinterpret_cast<uint32_t *>(Tt + toff(16 * bi + g8, cc, 64)) =
                    pack_bf16x2(acc[nt][0] * b0, acc[nt][1] * b1);
                *reinterpret_cast<uint32_t *>(Tt + toff(16 * bi + g8 + 8, cc, 64)) =
                    pack_bf16x2(acc[nt][2] * b0, acc[nt][3] * b1);
            }
        };
        // Below the diagonal, X_ij = -X_ii sum_{k=j}^{i-1} A_ik X_kj, merging 16 -> 32 -> 64.
        // The 32 x 32 halves: X_10 = -X_11 (A_10 X_00) (warp 0), X_32 = -X_33 (A_32 X_22) (warp 1)
        if (warp < 2) {
            const int i = warp == 0 ? 1 : 3, jj = i - 1;
            float *Y = Ys + warp * 16 * YS_LD;
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            mma16_tf32(acc, As + 16 * i * AS_LD + 16 * jj, AS_LD, Xs + 16 * jj * AS_LD + 16 * jj, AS_LD, g8, t4);
            store16(Y, YS_LD, acc, 1.f, g8, t4);
            __syncwarp();
            float xa[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            mma16_tf32(xa, Xs + 16 * i * AS_LD + 16 * i, AS_LD, Y, YS_LD, g8, t4);
            store16(Xs + 16 * i * AS_LD + 16 * jj, AS_LD, xa, -1.f, g8, t4);
            store_t(i, jj, xa, -1.f);
        }
        __syncthreads();
        // the lower-left 32 x 32 quarter, X_BA = -X_B (A_BA X_A) with A = rows 0-31, B = rows
        // 32-63; warp w takes block (i, j) = (2 + w / 2, w % 2): Y_ij = sum_k A_ik X_kj ...
        if (warp < 4) {
            const int i = 2 + (warp >> 1), jj = warp & 1;
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            if (jj == 0) {
                mma16_tf32(acc, As + 16 * i * AS_LD, AS_LD, Xs, AS_LD, g8, t4);
                mma16_tf32(acc, As + 16 * i * AS_LD + 16, AS_LD, Xs + 16 * AS_LD, AS_LD, g8, t4);
            } else {
                mma16_tf32(acc, As + 16 * i * AS_LD + 16, AS_LD, Xs + 16 * AS_LD + 16, AS_LD, g8, t4);
            }
            store16(Ys + warp * 16 * YS_LD, YS_LD, acc, 1.f, g8, t4);
        }
        __syncthreads();
        // ... then X_2j = -X_22 Y_2j and X_3j = -(X_32 Y_2j + X_33 Y_3j)
        if (warp < 4) {
            const int i = 2 + (warp >> 1), jj = warp & 1;
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            mma16_tf32(acc, Xs + 16 * i * AS_LD + 32, AS_LD, Ys + jj * 16 * YS_LD, YS_LD, g8, t4);
            if (i == 3) mma16_tf32(acc, Xs + 48 * AS_LD + 48, AS_LD, Ys + (2 + jj) * 16 * YS_LD, YS_LD, g8, t4);
            store_t(i, jj, acc, -1.f);
        }
    }
    fence_proxy_async_smem();  // T, Kt, Qt (GDN) are read by the tensor cores
    __syncthreads();

    // ---- [W | Ut] = [T; -] [Kt | V]: M = 128 (rows 0-63 used), N = 128 + 128, K = 64 ---------
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(sb + PA_KH + kk * 32, 16, 1024);
            const uint64_t bk = smem_desc_sw128(sb + PA_KQ + kk * 2048, 16384, 1024);
            const uint64_t bv = smem_desc_sw128(sb + PA_V + kk * 2048, 8192, 1024);
            umma_bf16(tmem, ad, bk, ID_WU, kk > 0 ? 1u : 0u);
            umma_bf16(tmem + 128, ad, bv, ID_WU, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_mma);
    }
    const uint32_t ph2 = fallback ? 0u : 1u;
    if (__syncthreads_or(!mbar_wait_bounded(bar_mma, ph2))) {
        abort_cta(bar_mma, ph2);
        return;
    }
    tc_fence_after();
    if ((warp & 3) < 2) {
        // token row r: warps 0, 1 take W (-W over the Kt rows of the [.; Qt] tile), warps 4, 5
        // take Ut (over the free V tile)
        const int r = 32 * (warp & 3) + lane;
        const bool w_side = warp < 4;
        uint8_t *dst = sm + (w_side ? PA_KQ : PA_V);
        const float sgn = w_side ? -1.f : 1.f;
        uint32_t d[32];
#pragma unroll
        for (int hq = 0; hq < 4; ++hq) {
            tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (w_side ? 0 : 128) + 32 * hq, d);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w[e] = pack_bf16x2(sgn * __uint_as_float(d[8 * u + 2 * e]),
                                       sgn * __uint_as_float(d[8 * u + 2 * e + 1]));
                *reinterpret_cast<uint4 *>(dst + (w_side ? toff(r, 32 * hq + 8 * u, 128)
                                                         : toff(r, 32 * hq + 8 * u, 64))) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        bulk_store(rec + REC_WQ, sb + PA_KQ, 32768);
        bulk_store(rec + REC_UT, sb + PA_V, 16384);
        bulk_commit_group();
        bulk_wait_group_read0();  // shared memory must outlive the copies' reads
    }
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kPrepTmemCols);
    }
}

// ================================ pass B ==================================================
// One CTA per (sequence, head, half of d_v): 64 state columns, the records streamed through a
// 3-stage ring (each CTA reads the whole record but its own half of Ut).
constexpr int kScanThreads = 384;  // 12 warps
constexpr int kSplitV = 2;
constexpr int kDV = kD / kSplitV;  // 64 state columns per CTA
constexpr int kStages = 3;
constexpr int kStateWarps = 8;     // warp w: TMEM lanes 32 (w % 4) .., columns 32 (w / 4) ..
constexpr int kWarpProducer = 8, kWarpMma = 9;  // 10-11: outputs
constexpr uint32_t ST_WQ = 0, ST_KC = 32768, ST_P = 49152, ST_GAM = 57344, ST_UT = 57856,
                   ST_BYTES = 66560;  // one stage (1 KiB multiple)
constexpr uint32_t ST_LOAD = ST_UT - ST_GAM + 57344 + kDV * kC * 2;  // bytes copied per stage
constexpr uint32_t SB_M = kStages * ST_BYTES;  // M bf16 [128 d_k][64 d_v], MN-major B operand
constexpr uint32_t SB_U = SB_M + 16384;        // U bf16 [64 tok][64 d_v], MN-major B operand
constexpr uint32_t SB_SMALL = SB_U + 8192;     // barriers, TMEM slot, abort flag
constexpr uint32_t SB_SMEM = SB_SMALL + 256 + 1024;
constexpr uint32_t kScanTmemCols = 256;  // D_UO x2 (0-63, 64-127), D_S (128-191)
constexpr uint32_t ID_64 = idesc_bf16(128, 64, 0, 1);  // A K-major, B MN-major
constexpr uint32_t ID_KC = idesc_bf16(128, 64, 1, 1);  // A MN-major (Kc^T), B MN-major
static_assert(ST_UT + kDV * kC * 2 <= ST_BYTES && ST_BYTES % 1024 == 0, "stage");
static_assert(ST_LOAD == 57344 + 512 + 8192, "bytes per stage");
static_assert(SB_SMEM <= 232448, "shared memory per CTA");

enum { BAR_FULL0 = 0, BAR_EMPTY0 = BAR_FULL0 + kStages, BAR_M = BAR_EMPTY0 + kStages, BAR_UO,
       BAR_U, BAR_S, BAR_OFULL0, BAR_TEMPTY0 = BAR_OFULL0 + 2, BAR_FINAL = BAR_TEMPTY0 + 2,
       N_BARS };

__global__ void __launch_bounds__(kScanThreads, 1) prefill_scan_kernel(const PrefillScanArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SB_SMALL);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + SB_SMALL + 8 * N_BARS);
    volatile int *s_abort = reinterpret_cast<volatile int *>(sm + SB_SMALL + 8 * N_BARS + 4);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x / kSplitV, sv = blockIdx.x - bh * kSplitV;
    const int b = bh / a.H, h = bh - b * a.H;
    const int T = a.T;
    const int nseg = a.n_seg;

    if (tid == 0) {
        for (int i = 0; i < N_BARS; ++i) {
            const bool by_threads = i == BAR_M || i == BAR_U || i == BAR_TEMPTY0 || i == BAR_TEMPTY0 + 1;
            mbar_init(bar(i), i == BAR_M ? kStateWarps : (i == BAR_U ? kStateWarps / 2 : (by_threads ? 2 : 1)));
        }
        fence_barrier_init();
        *s_abort = 0;
    }
    griddep_launch_dependents();
    griddep_wait();  // the records are the prep pass's output
    const int slot = a.slots ? a.slots[b] : b;
    const bool slot_ok = slot >= 0 && slot < a.n_slots;
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), kScanTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (!slot_ok) {
        if (tid == 0) atomicOr(&g_err, HMD_DEVERR_SLOT);
        if (warp == 0) {
            __syncwarp();
            tmem_dealloc(*tmem_slot, kScanTmemCols);
        }
        return;
    }
    const uint32_t tmem = *tmem_slot;
    float *Mg = a.state + ((size_t)slot * a.H + h) * kD * kD + sv * kDV;

    // bounded wait that also gives up once another thread of the CTA has given up. A warp that
    // goes on to a tcgen05 .sync.aligned instruction (a TMEM load) takes the decision as one
    // (__all_sync), so the instruction always runs converged.
    auto wait = [&](int i, uint32_t parity) -> bool {
        const uint32_t bb = bar(i);
        if (mbar_try_wait(bb, parity)) return true;
        const unsigned long long t0 = globaltimer_ns();
        while (true) {
            if (mbar_try_wait(bb, parity)) return true;
            if (*s_abort) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *s_abort = 1;
                atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
                return false;
            }
        }
    };

    int issued = 0;  // producer: chunks issued
    if (warp == kWarpProducer) {
        // ---- producer: chunk c's record (its half of Ut) -> stage c % kStages ---------------
        if (lane == 0) {
            for (int c = 0; c < nseg; ++c) {
                const int s = c % kStages;
                if (c >= kStages && !wait(BAR_EMPTY0 + s, ((c / kStages) - 1) & 1)) break;
                const uint8_t *rec = record(a, bh, c);
                const uint32_t st = sb + s * ST_BYTES;
                mbar_arrive_expect_tx(bar(BAR_FULL0 + s), ST_LOAD);
                bulk_load(st + ST_WQ, rec + REC_WQ, 57344, bar(BAR_FULL0 + s));  // [-W; Qt], Kc, P
                bulk_load(st + ST_GAM, rec + REC_GAM, 512, bar(BAR_FULL0 + s));
                bulk_load(st + ST_UT, rec + REC_UT + sv * (kDV * kC * 2), kDV * kC * 2,
                          bar(BAR_FULL0 + s));
                ++issued;
            }
        }
    } else if (warp == kWarpMma) {
        // ---- the tensor-core products -----------------------------------------------------
        if (lane == 0) {
            // descriptors: the address field is the byte address / 16, so an offset is added as
            // offset / 16 (every address here is below 256 KiB: no carry out of the field)
            const uint64_t d_wq = smem_desc_sw128(sb + ST_WQ, 16, 1024);
            const uint64_t d_p = smem_desc_sw128(sb + ST_P - 8192, 16, 1024);
            const uint64_t d_kc = smem_desc_sw128(sb + ST_KC, 8192, 1024);
            const uint64_t d_m = smem_desc_sw128(sb + SB_M, 16384, 1024);
            const uint64_t d_u = smem_desc_sw128(sb + SB_U, 8192, 1024);
            for (int c = 0; c < nseg; ++c) {
                const int s = c % kStages, u = c & 1;
                const uint64_t so = (uint64_t)((s * ST_BYTES) >> 4);
                if (!wait(BAR_FULL0 + s, (c / kStages) & 1)) break;
                if (c >= 2 && !wait(BAR_TEMPTY0 + u, ((c - 2) >> 1) & 1)) break;
                if (!wait(BAR_M, c & 1)) break;
                tc_fence_after();
                // D_UO = [-W; Qt] M
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    umma_bf16(tmem + kDV * u, d_wq + so + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                              d_m + ((kk * 2048) >> 4), ID_64, kk > 0 ? 1u : 0u);
                umma_commit(bar(BAR_UO));
                if (!wait(BAR_U, c & 1)) break;
                tc_fence_after();
                // D_S = Kc^T U first (the state waits for it), then D_UO += [- ; P] U (rows
                // 64-127: O; rows 0-63 read the Kc tile's second half and land on lanes whose
                // -W M was consumed already)
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    umma_bf16(tmem + 2 * kDV, d_kc + so + ((kk * 2048) >> 4), d_u + ((kk * 2048) >> 4),
                              ID_KC, kk > 0 ? 1u : 0u);
                umma_commit(bar(BAR_S));
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    umma_bf16(tmem + kDV * u, d_p + so + ((kk * 32) >> 4), d_u + ((kk * 2048) >> 4),
                              ID_64, 1u);
                umma_commit(bar(BAR_OFULL0 + u));
                umma_commit(bar(BAR_EMPTY0 + s));
            }
            umma_commit(bar(BAR_FINAL));  // every product issued has completed once this fires
        }
    } else if (warp >= 10) {
        // ---- outputs: O rows from TMEM lanes 64-127 ----------------------------------------
        const int r = 32 * (warp & 3) - 64 + lane;  // token row 0..63
        __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o);
        for (int c = 0; c < nseg; ++c) {
            const int u = c & 1;
            if (!__all_sync(0xffffffffu, wait(BAR_OFULL0 + u, (c >> 1) & 1))) break;
            tc_fence_after();
            const int t0 = (a.chunk_begin + c) * kC;
            const int n = min(kC, T - t0);
            uint4 *orow = reinterpret_cast<uint4 *>(og + (((size_t)b * T + t0 + r) * a.H + h) * kD + sv * kDV);
            uint32_t d[64];
            tmem_ld64(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + kDV * u, d);
            tmem_wait_ld();
            if (r < n) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint4 w;
                    w.x = pack_bf16x2(a.scale * __uint_as_float(d[8 * q]), a.scale * __uint_as_float(d[8 * q + 1]));
                    w.y = pack_bf16x2(a.scale * __uint_as_float(d[8 * q + 2]), a.scale * __uint_as_float(d[8 * q + 3]));
                    w.z = pack_bf16x2(a.scale * __uint_as_float(d[8 * q + 4]), a.scale * __uint_as_float(d[8 * q + 5]));
                    w.w = pack_bf16x2(a.scale * __uint_as_float(d[8 * q + 6]), a.scale * __uint_as_float(d[8 * q + 7]));
                    orow[q] = w;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BAR_TEMPTY0 + u));
        }
    } else if (warp < kStateWarps) {
        // ---- state: thread = row i of d_k, 32 of this CTA's 64 columns --------------------
        // Per chunk c: the warps over rows 0-63 form U from D_UO; all wait for D_S and update
        // M <- e^G_C(c) M + D_S, then write bf16(M) for chunk c + 1 right away (chunk c's first
        // product, the last reader of that tile, has completed by then).
        const int quad = warp & 3, half = warp >> 2;
        const int i = 32 * quad + lane, col0 = 32 * half;
        const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
        float st[32];
        {
            const float4 *src = reinterpret_cast<const float4 *>(Mg + (size_t)i * kD + col0);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 v = src[q];
                st[4 * q] = v.x; st[4 * q + 1] = v.y; st[4 * q + 2] = v.z; st[4 * q + 3] = v.w;
            }
        }
        uint8_t *mrow = sm + SB_M + i * 128;
        // e^G_C of chunk c, read before this thread lets chunk c's products start (its stage
        // cannot be refilled before then); then bf16(M) -> the B operand, and arrive
        float gam = 0.f;
        auto publish_m = [&](int c) -> bool {
            const int s = c % kStages;
            if (!__all_sync(0xffffffffu, wait(BAR_FULL0 + s, (c / kStages) & 1))) return false;
            gam = reinterpret_cast<const float *>(sm + s * ST_BYTES + ST_GAM)[i];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int chunk = 4 * half + q;
                *reinterpret_cast<uint4 *>(mrow + ((chunk ^ (i & 7)) << 4)) =
                    make_uint4(pack_bf16x2(st[8 * q], st[8 * q + 1]), pack_bf16x2(st[8 * q + 2], st[8 * q + 3]),
                               pack_bf16x2(st[8 * q + 4], st[8 * q + 5]), pack_bf16x2(st[8 * q + 6], st[8 * q + 7]));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BAR_M));
            return true;
        };
        bool ok = nseg > 0 && publish_m(0);
        for (int c = 0; ok && c < nseg; ++c) {
            const int s = c % kStages, u = c & 1;
            if (quad < 2) {
                // U = Ut + (-W M) for token row i, bf16 into the U operand; Ut is read before the
                // product lands
                const uint8_t *utrow = sm + s * ST_BYTES + ST_UT + i * 128;
                uint4 ut[4];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    ut[q] = *reinterpret_cast<const uint4 *>(utrow + (((4 * half + q) ^ (i & 7)) << 4));
                if (!__all_sync(0xffffffffu, wait(BAR_UO, c & 1))) break;
                tc_fence_after();
                uint32_t d[32];
                tmem_ld32(tmem + lane_base + kDV * u + col0, d);
                tmem_wait_ld();
                uint8_t *urow = sm + SB_U + i * 128;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t uw[4] = {ut[q].x, ut[q].y, ut[q].z, ut[q].w};
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[e] = pack_bf16x2(bf16_lo(uw[e]) + __uint_as_float(d[8 * q + 2 * e]),
                                           bf16_hi(uw[e]) + __uint_as_float(d[8 * q + 2 * e + 1]));
                    *reinterpret_cast<uint4 *>(urow + (((4 * half + q) ^ (i & 7)) << 4)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BAR_U));
            }
            // M <- e^G_C M + Kc^T U
            if (!__all_sync(0xffffffffu, wait(BAR_S, c & 1))) break;
            tc_fence_after();
            {
                uint32_t d[32];
                tmem_ld32(tmem + lane_base + 2 * kDV + col0, d);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) st[e] = fmaf(gam, st[e], __uint_as_float(d[e]));
            }
            tc_fence_before();
            if (c + 1 < nseg && !publish_m(c + 1)) break;
        }
        if (!*s_abort) {
            float4 *dst = reinterpret_cast<float4 *>(Mg + (size_t)i * kD + col0);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(st[4 * q], st[4 * q + 1], st[4 * q + 2], st[4 * q + 3]);
        }
    }

    // ---- teardown: every copy and product in flight ends (bounded) before the memory goes ----
    if (warp == kWarpProducer && lane == 0 && *s_abort) {
        // the last stages issued may not have been consumed: let their copies land
        for (int c = std::max(0, issued - kStages); c < issued; ++c)
            (void)mbar_wait_bounded(bar(BAR_FULL0 + c % kStages), (c / kStages) & 1);
    }
    if (warp == kWarpMma && lane == 0) (void)mbar_wait_bounded(bar(BAR_FINAL), 0);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kScanTmemCols);
    }
}

}  // namespace

bool delta_prefill_scan_supported(int dk, int dv, bool bf16, int chunk) {
    return bf16 && dk == kD && dv == kD && chunk == kC;
}

size_t delta_prefill_scan_record_bytes() { return REC_BYTES; }

cudaError_t launch_delta_prefill_scan(const DeltaPrefillArgs &a, void *ws, size_t ws_bytes,
                                      cudaStream_t s) {
    const cudaError_t attr = once_per_device([] {
        cudaError_t e = cudaSuccess;
        for (auto k : {prefill_prep_kernel<true, false>, prefill_prep_kernel<true, true>,
                       prefill_prep_kernel<false, false>, prefill_prep_kernel<false, true>})
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PA_SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)SB_SMEM);
        return e;
    });
    if (attr != cudaSuccess) return attr;
    const long long bhs = (long long)a.B * a.H;
    const int n_chunks = (a.T + kC - 1) / kC;
    if (bhs <= 0 || n_chunks <= 0) return cudaSuccess;
    const long long fit = (long long)(ws_bytes / ((size_t)bhs * REC_BYTES));
    if (fit < 1 || (reinterpret_cast<uintptr_t>(ws) & 15)) return cudaErrorInvalidValue;
    const int seg = (int)std::min<long long>(n_chunks, fit);
    CUtensorMap tmq, tmk, tmv, tmg;
    if (!make_tmap_bthd(&tmq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q, a.B, a.T, a.H, kD, 64, true) ||
        !make_tmap_bthd(&tmk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.k, a.B, a.T, a.H, kD, 64, true) ||
        !make_tmap_bthd(&tmv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.v, a.B, a.T, a.H, kD, 64, true))
        return cudaErrorInvalidValue;
    if (a.kind == HMD_KDA) {
        if (!make_tmap_bthd(&tmg, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.log_gate, a.B, a.T, a.H, kD,
                            32, true))
            return cudaErrorInvalidValue;
    } else {
        tmg = tmq;  // not read
    }
    PrefillScanArgs p;
    p.q = a.q; p.k = a.k; p.v = a.v; p.beta = a.beta; p.log_gate = a.log_gate;
    p.state = a.state; p.slots = a.slots; p.n_slots = a.n_slots; p.o = a.o;
    p.B = a.B; p.T = a.T; p.H = a.H; p.scale = a.scale; p.ws = ws; p.act = a.act;
    p.prefetch_stride = 2 * once_per_device([] {  // resident prep CTAs: two per SM
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            return v;
        cudaGetLastError();
        return 148;
    });
    for (int cb = 0; cb < n_chunks; cb += seg) {
        p.chunk_begin = cb;
        p.n_seg = std::min(seg, n_chunks - cb);
        const unsigned grid_a = (unsigned)(bhs * p.n_seg);
        const bool fused = a.act.A_log != nullptr;
        cudaError_t e = launch_pdl(a.kind == HMD_KDA ? (fused ? prefill_prep_kernel<true, true> : prefill_prep_kernel<true, false>)
                                                     : (fused ? prefill_prep_kernel<false, true> : prefill_prep_kernel<false, false>),
                                   dim3(grid_a), dim3(kPrepThreads), PA_SMEM, s, tmq, tmk, tmv, tmg, p);
        if (e != cudaSuccess) return e;
        e = launch_pdl(prefill_scan_kernel, dim3((unsigned)(bhs * kSplitV)), dim3(kScanThreads),
                       SB_SMEM, s, p);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

uint32_t delta_prefill_scan_read_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_err, sizeof v) != cudaSuccess) return 0;
    if (clear && v) {
        const unsigned int z = 0;
        cudaMemcpyToSymbol(g_err, &z, sizeof z);
    }
    return v;
}

}  // namespace hmd

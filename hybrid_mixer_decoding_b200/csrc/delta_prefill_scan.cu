// Chunked delta-rule prefill in two passes, bf16 activations, fp32 state and accumulation,
// d_k = d_v = 128, chunk C = 64.
//
// Chunk algebra: the standard WY / UT-transform rewriting of the gated delta rule for the GDN and
// KDA mixers of "Super Apriel: One Checkpoint, Many Speeds" (abstract; gist.science technical
// summary, section 2a). For a chunk with start state M ([d_k][d_v] fp32) and G the per-channel
// cumulative log-gate inside the chunk (G_C its last row):
//   Kt = k e^G, Kh = k e^-G, Qt = q e^G, Kc = k e^(G_C - G)
//   A = beta_r (Kt Kh^T)_{rs} (s < r),  P = (Qt Kh^T)_{rs} (s <= r)
//   T = (I + A)^-1 Diag(beta),  W = T Kt,  Ut = T V
//   U = Ut - W M,  O = Qt M + P U,  M_next = Diag(e^{G_C}) M + Kc^T U
// Everything up to W and Ut depends only on the chunk's own inputs; only the last line carries
// the state from chunk to chunk.
//
// Pass A (prefill_prep_kernel): one CTA per (sequence, head, chunk), all chunks at once, on the
// 5th-generation tensor cores. TMA brings the chunk's q, k, v (and KDA log-gates) into shared
// memory in the 128-byte swizzled layout the tensor cores read; the CTA forms the gate factors,
// then [Kt; Qt] Kh^T as ONE M = 128 tcgen05.mma product into TMEM (rows 0-63 give A, rows 64-127
// give P), the blocked fp32 UT solve on the CUDA cores, and W^T, Ut^T as two M = 128 products
// that read Kt and V MN-major. It writes one record per chunk: Qt, Kc, P, and -W^T, Ut^T (rows of
// d_k / d_v, as the TMEM read-back delivers them), all bf16 in the 128-byte XOR-swizzled tile
// layout pass B reads with ldmatrix, and e^{G_C} (fp32).
// Pass B (prefill_scan_kernel, mma.sync m16n8k16): one CTA per (sequence, head, half of d_v)
// walks the chunks in order. Each chunk's whole record arrives by one bulk copy into a 2-stage
// shared-memory ring while the chunk before it computes; the state half lives in registers as MMA accumulator fragments.
// Per chunk it does only the state-dependent products (U, O, state update): 7.3 MFLOP of the
// chunk's 11.5 per head, split over two CTAs.
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
constexpr int kThreads = 256;       // pass B
constexpr int kPrepThreads = 256;   // pass A: 8 warps, two CTAs per SM
constexpr int kSplitV = 2;             // pass B: CTAs per (sequence, head), each d_v / 2 columns
constexpr int kDV = kD / kSplitV;      // 64 columns of d_v per pass-B CTA

// ---- the per-chunk record (bytes) ----------------------------------------------------------
constexpr uint32_t REC_QT = 0;         // Qt  bf16 [64][128], swizzled halves
constexpr uint32_t REC_NW = 16384;     // -W^T bf16 [128 d_k][64 tokens] (tile of 128 rows)
constexpr uint32_t REC_KC = 32768;     // Kc  bf16 [64][128]
constexpr uint32_t REC_P = 49152;      // P   bf16 [64][64]
constexpr uint32_t REC_GAM = 57344;    // e^{G_C} fp32 [128]
constexpr uint32_t REC_HEAD = 57856;   // bytes above
constexpr uint32_t REC_UT = 57856;     // Ut^T bf16 [128 d_v][64 tokens] (tile of 128 rows)
constexpr uint32_t REC_BYTES = REC_UT + kC * kD * 2;  // 74240
static_assert(REC_HEAD % 16 == 0 && REC_BYTES % 16 == 0, "bulk copies need 16-byte sizes");

// ---- pass A shared memory (bytes from a 1024-aligned base) ---------------------------------
constexpr uint32_t A_KQ = 0;           // [Kt; Qt], the K-major A operand of one M = 128 product:
                                       //   two 64-column halves of 128 rows (16 KiB each), Kt in
                                       //   rows 0-63, q then Qt in rows 64-127; at the end -W
                                       //   (record layout) in the Kt rows; Kt is also read
                                       //   MN-major (halves 16 KiB apart)
constexpr uint32_t A_KH = 32768;       // k, then Kh [64][128] (K-major B operand); then P, e^{G_C}
constexpr uint32_t A_V = 49152;        // v [64][128] (MN-major A operand); at the end -W^T
constexpr uint32_t A_G = 65536;        // KDA log-gates -> in-chunk prefix, fp32 [4][64][32]
constexpr uint32_t A_AS = 65536;       // after the gate pass: A fp32 [64][68], then T bf16
constexpr uint32_t A_XS = 82944;       // X fp32 [64][68]
constexpr uint32_t A_YS = 100352;      // Y fp32 [3][16][20]
constexpr uint32_t A_UT = 65536;       // at the end: Ut^T bf16 (record layout, 16 KiB)
constexpr uint32_t A_SMALL = 104192;
constexpr uint32_t S_BETA = 0, S_QOFF = 256, S_LGP = 1280, S_WSUM = 1536, S_EGC = 1552,
                   S_BAR = 2064, S_TMEM = 2080, S_NRM = 2112, S_SIZE = 2624;
constexpr uint32_t A_SMEM = A_SMALL + S_SIZE + 1024;
constexpr uint32_t A_T = A_KQ + 8192;  // T bf16 [64][64]: the Qt rows of the first half
constexpr int AS_LD = 68;
constexpr int YS_LD = 20;
constexpr uint32_t kPrepTmemCols = 128;
constexpr uint32_t ID_AP = idesc_bf16(128, 64, 0, 0);  // [Kt; Qt] Kh^T: both operands K-major
constexpr uint32_t ID_WU = idesc_bf16(128, 64, 1, 0);  // Kt^T T^T, V^T T^T: A MN-major
static_assert(A_G + kC * kD * 4 <= A_YS, "log-gate staging fits the A/X region");
static_assert(A_UT + kC * kD * 2 <= A_YS, "Ut fits the A/X region");
static_assert(S_QOFF + (kPrepThreads / kD) * kD * 4 <= S_LGP, "gate part sums fit");
static_assert(S_BAR % 8 == 0 && S_TMEM + 4 <= S_SIZE, "small area");

// ---- pass B shared memory ----------------------------------------------------------------
constexpr uint32_t B_STAGE = 74752;        // one whole record (one bulk copy), padded to 1 KiB
constexpr uint32_t B_M = 2 * B_STAGE;      // M bf16 [128][64], two buffers (chunk parity)
constexpr uint32_t B_U = B_M + 2 * 16384;  // U bf16 [64][64], two buffers
constexpr uint32_t B_BAR = B_U + 2 * 8192;
constexpr uint32_t B_SMEM = B_BAR + 64 + 1024;

// byte offset of element (row, col) of a tile whose halves (64 columns each) hold `rows` rows
__device__ __forceinline__ uint32_t toff(int row, int col, int rows) {
    return (uint32_t)((col >> 6) * rows * 128 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                      ((col & 7) << 1));
}

// float index of log-gate (row r, channel i) in the staged KDA gate tile: four TMA boxes of
// [64 rows][32 channels]
__device__ __forceinline__ int gidx(int r, int i) { return (i >> 5) * 2048 + r * 32 + (i & 31); }

__device__ __forceinline__ void st_bf16x2(uint8_t *base, uint32_t off, float lo, float hi) {
    *reinterpret_cast<uint32_t *>(base + off) = pack_bf16x2(lo, hi);
}

__device__ __forceinline__ uint8_t *record(const PrefillScanArgs &a, int bh, int c) {
    return static_cast<uint8_t *>(a.ws) + ((size_t)bh * a.n_seg + c) * REC_BYTES;
}

// ================================ pass A ==================================================
constexpr int pow2_floor(int x) { return x >= 2 ? 2 * pow2_floor(x / 2) : 1; }

// One level of the blocked inverse X = (I + A)^-1 (16x16 blocks): the blocks (i, j) with
// i - j = L. Y_ij = sum_{k=j}^{i-1} A_ik X_kj, then X_ij = -X_ii Y_ij. Each (block, row,
// 4-column group) is shared by as many threads as the block has to spare (a power of two);
// they split the sums and combine them by shuffles.
template <int L>
__device__ __forceinline__ void solve_level(const float *As, float *Xs, float *Ys, int tid,
                                            uint8_t *Tt, const float *sbeta) {
    constexpr int NB = 4 - L;                                  // blocks on this diagonal
    constexpr int TPI = pow2_floor(kPrepThreads / (NB * 64));  // threads per (block, row, group)
    constexpr int KPT = 16 * L / TPI;  // terms of Y per thread
    constexpr int XPT = 16 / TPI;      // terms of X_ii Y_ij per thread
    const bool active = tid < NB * 64 * TPI;  // whole warps
    const int item = tid / TPI, part = tid % TPI;
    const int j = item >> 6, r = (item >> 2) & 15, cg = item & 3, i = j + L;
    if (active) {
        const float *arow = As + (i * 16 + r) * AS_LD;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int kk = 0; kk < KPT; ++kk) {
            const int k = j * 16 + part * KPT + kk;
            const float av = arow[k];
            const float4 xv = *reinterpret_cast<const float4 *>(Xs + k * AS_LD + j * 16 + cg * 4);
            acc.x += av * xv.x; acc.y += av * xv.y; acc.z += av * xv.z; acc.w += av * xv.w;
        }
#pragma unroll
        for (int m = 1; m < TPI; m <<= 1) {
            acc.x += __shfl_xor_sync(0xffffffffu, acc.x, m);
            acc.y += __shfl_xor_sync(0xffffffffu, acc.y, m);
            acc.z += __shfl_xor_sync(0xffffffffu, acc.z, m);
            acc.w += __shfl_xor_sync(0xffffffffu, acc.w, m);
        }
        if (part == 0) *reinterpret_cast<float4 *>(Ys + (j * 16 + r) * YS_LD + cg * 4) = acc;
    }
    __syncthreads();
    if (active) {
        const float *xrow = Xs + (i * 16 + r) * AS_LD + i * 16;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int ss = 0; ss < XPT; ++ss) {
            const int s2 = part * XPT + ss;
            const float xv = s2 <= r ? xrow[s2] : 0.f;  // X_ii is lower triangular
            const float4 yv = *reinterpret_cast<const float4 *>(Ys + (j * 16 + s2) * YS_LD + cg * 4);
            acc.x += xv * yv.x; acc.y += xv * yv.y; acc.z += xv * yv.z; acc.w += xv * yv.w;
        }
#pragma unroll
        for (int m = 1; m < TPI; m <<= 1) {
            acc.x += __shfl_xor_sync(0xffffffffu, acc.x, m);
            acc.y += __shfl_xor_sync(0xffffffffu, acc.y, m);
            acc.z += __shfl_xor_sync(0xffffffffu, acc.z, m);
            acc.w += __shfl_xor_sync(0xffffffffu, acc.w, m);
        }
        if (part == 0) {
            *reinterpret_cast<float4 *>(Xs + (i * 16 + r) * AS_LD + j * 16 + cg * 4) =
                make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
            // the same four entries of T = X Diag(beta), bf16 (8 bytes of one 16-byte chunk)
            const int s0 = j * 16 + cg * 4;
            *reinterpret_cast<uint2 *>(Tt + toff(i * 16 + r, s0, 64)) =
                make_uint2(pack_bf16x2(-acc.x * sbeta[s0], -acc.y * sbeta[s0 + 1]),
                           pack_bf16x2(-acc.z * sbeta[s0 + 2], -acc.w * sbeta[s0 + 3]));
        }
    }
    __syncthreads();
}

template <bool KDA>
__global__ void __launch_bounds__(kPrepThreads, 2)
prefill_prep_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmg,
                    const PrefillScanArgs a) {
    constexpr int NT = kPrepThreads;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    float *Gs = reinterpret_cast<float *>(sm + A_G);
    float *As = reinterpret_cast<float *>(sm + A_AS);
    float *Xs = reinterpret_cast<float *>(sm + A_XS);
    float *Ys = reinterpret_cast<float *>(sm + A_YS);
    float *sbeta = reinterpret_cast<float *>(sm + A_SMALL + S_BETA);  // [64]
    float *qoff = reinterpret_cast<float *>(sm + A_SMALL + S_QOFF);   // [NQ][128] KDA: gate sums
                                                                       //   of the row parts, then
                                                                       //   their exclusive prefix
    float *lgp = reinterpret_cast<float *>(sm + A_SMALL + S_LGP);     // [64] GDN log-gate prefix
    float *wsum = reinterpret_cast<float *>(sm + A_SMALL + S_WSUM);   // [2]
    float *egc = reinterpret_cast<float *>(sm + A_SMALL + S_EGC);     // [128] e^{G_C}
    float *nrm = reinterpret_cast<float *>(sm + A_SMALL + S_NRM);     // [2][64] 1/|q|, 1/|k|
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + A_SMALL + S_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + A_SMALL + S_TMEM);

    constexpr int NQ = NT / kD;       // KDA gate prefix: row parts per channel
    constexpr int RPQ = kC / NQ;      // rows per part
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x / a.n_seg, c = blockIdx.x - bh * a.n_seg;
    const int b = bh / a.H, h = bh - b * a.H;
    const int T = a.T;
    const int t0 = (a.chunk_begin + c) * kC;
    const int n = min(kC, T - t0);
    uint8_t *rec = record(a, bh, c);
    const uint32_t bar_in = smem_u32(&bars[0]), bar_mma = smem_u32(&bars[1]);

    if (tid == 0) {
        mbar_init(bar_in, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&tmq);
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        if constexpr (KDA) prefetch_tmap(&tmg);
    }
    griddep_launch_dependents();
    griddep_wait();  // the inputs may come from the previous kernel
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), kPrepTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Abort after a wait gave up: let the copies and products in flight end (bounded), free
    // the tensor memory, report. Every thread of the CTA takes this path together.
    auto abort_cta = [&](uint32_t bar, uint32_t parity) {
        if (tid == 0) {
            atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
            (void)mbar_wait_bounded(bar, parity);
            bulk_wait_group_read0();
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            __syncwarp();
            tc_fence_after();
            tmem_dealloc(tmem, kPrepTmemCols);
        }
    };

    // ---- inputs: q (into the Qt rows), k (into the Kh slot), v, KDA log-gates by TMA; rows
    //      past the end of the sequence read as zero. beta and the GDN log-gates by plain loads.
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_in, (KDA ? 10u : 6u) * 8192u);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(sb + A_KQ + hf * 16384 + 8192, &tmq, bar_in, hf * 64, h, t0, b);
            tma_load_4d(sb + A_KH + hf * 8192, &tmk, bar_in, hf * 64, h, t0, b);
            tma_load_4d(sb + A_V + hf * 8192, &tmv, bar_in, hf * 64, h, t0, b);
        }
        if constexpr (KDA) {
#pragma unroll
            for (int j = 0; j < 4; ++j) tma_load_4d(sb + A_G + j * 8192, &tmg, bar_in, j * 32, h, t0, b);
        }
    }
    const bool fused = a.act.A_log != nullptr;  // raw projections: activate them here
    const float rate = fused ? expf(a.act.A_log[h]) : 0.f;
    if (tid < kC) {
        const size_t tok = ((size_t)b * T + t0 + tid) * a.H + h;
        float bt = tid < n ? a.beta[tok] : 0.f;
        if (fused && tid < n) bt = 1.f / (1.f + expf(-bt));
        sbeta[tid] = bt;
        if constexpr (!KDA) {
            float x = tid < n ? a.log_gate[tok] : 0.f;
            if (fused && tid < n) x = -rate * hmd_softplus(x + a.act.dt_bias[h]);
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            if (lane == 31) wsum[warp] = x;
            lgp[tid] = x;
        }
    }
    if (__syncthreads_or(!mbar_wait_bounded(bar_in, 0))) {
        abort_cta(bar_in, 0);
        return;
    }

    // ---- gate prefix G (log domain): KDA per channel in place within NQ row parts, plus the
    //      parts' exclusive prefix; GDN per token -------------------------------------------------
    if (fused) {  // 1/|q| and 1/|k| of each row: 4 threads per row, 32 channels each
        static_assert(NT == 4 * kC, "four threads per row");
        const int r = tid >> 2, qq = tid & 3;
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            const int c0 = qq * 32 + c4 * 8;
            const uint4 qv = *reinterpret_cast<const uint4 *>(sm + A_KQ + toff(64 + r, c0, 128));
            const uint4 kv = *reinterpret_cast<const uint4 *>(sm + A_KH + toff(r, c0, 64));
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
    if constexpr (KDA) {
        if (fused) {  // log-gates from the staged logits, in place, 4 channels per item
            const float *db = a.act.dt_bias + (size_t)h * kD;
#pragma unroll
            for (int j = 0; j < kC * kD / 4 / NT; ++j) {
                const int e = 4 * (tid + j * NT);
                const int r = (e & 2047) >> 5, ch = (e >> 11) * 32 + (e & 31);  // gidx inverse
                float4 x = *reinterpret_cast<const float4 *>(Gs + e);
                const float4 bb = make_float4(db[ch], db[ch + 1], db[ch + 2], db[ch + 3]);
                const bool live = r < n;  // rows past the sequence read as zero and stay zero
                x.x = live ? -rate * hmd_softplus(x.x + bb.x) : 0.f;
                x.y = live ? -rate * hmd_softplus(x.y + bb.y) : 0.f;
                x.z = live ? -rate * hmd_softplus(x.z + bb.z) : 0.f;
                x.w = live ? -rate * hmd_softplus(x.w + bb.w) : 0.f;
                *reinterpret_cast<float4 *>(Gs + e) = x;
            }
            __syncthreads();
        }
        const int i = tid & (kD - 1), qr = tid >> 7;
        float *gcol = Gs + gidx(0, i);
        float run = 0.f;
#pragma unroll
        for (int r = RPQ * qr; r < RPQ * qr + RPQ; ++r) {
            run += gcol[r * 32];
            gcol[r * 32] = run;
        }
        qoff[qr * kD + i] = run;
        __syncthreads();
        if (qr == 0) {
            float acc = 0.f;
#pragma unroll
            for (int q2 = 0; q2 < NQ; ++q2) {
                const float part = qoff[q2 * kD + i];
                qoff[q2 * kD + i] = acc;
                acc += part;
            }
            egc[i] = __expf(acc);
            if (acc < kPrefillGateFloor) atomicOr(&g_err, HMD_DEVERR_GATE);
        }
    } else {
        if (tid < kC) lgp[tid] += (warp == 1 ? wsum[0] : 0.f);
        __syncthreads();
        if (tid < kD) egc[tid] = __expf(lgp[kC - 1]);
        if (tid == 0 && lgp[kC - 1] < kPrefillGateFloor) atomicOr(&g_err, HMD_DEVERR_GATE);
    }
    __syncthreads();

    // ---- gate factors, 8 channels of one row per item: Kt, Qt, Kh (shared memory), Kc -------
    //      (record), with e^{G_C - G} = e^{G_C} e^-G <= 1
    {
        uint8_t *kc = rec + REC_KC;
#pragma unroll
        for (int j = 0; j < kC * kD / 8 / NT; ++j) {
            const int idx = tid + j * NT, r = idx >> 4, c0 = (idx & 15) * 8;
            const uint32_t o = toff(r, c0, 64);
            const uint32_t okt = A_KQ + toff(r, c0, 128), oqt = A_KQ + toff(64 + r, c0, 128);
            const uint4 qr = *reinterpret_cast<const uint4 *>(sm + oqt);
            const uint4 kr = *reinterpret_cast<const uint4 *>(sm + A_KH + o);
            float G[8];
            if constexpr (KDA) {
                const float4 g0 = *reinterpret_cast<const float4 *>(Gs + gidx(r, c0));
                const float4 g1 = *reinterpret_cast<const float4 *>(Gs + gidx(r, c0) + 4);
                const float4 f0 = *reinterpret_cast<const float4 *>(qoff + (r / RPQ) * kD + c0);
                const float4 f1 = *reinterpret_cast<const float4 *>(qoff + (r / RPQ) * kD + c0 + 4);
                G[0] = g0.x + f0.x; G[1] = g0.y + f0.y; G[2] = g0.z + f0.z; G[3] = g0.w + f0.w;
                G[4] = g1.x + f1.x; G[5] = g1.y + f1.y; G[6] = g1.z + f1.z; G[7] = g1.w + f1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) G[e] = lgp[r];
            }
            const uint32_t qw[4] = {qr.x, qr.y, qr.z, qr.w};
            const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
            const float fq = fused ? nrm[r] : 1.f, fk = fused ? nrm[kC + r] : 1.f;
            uint32_t kt[4], qt[4], kh[4], kcw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float ea = __expf(G[2 * e]), eb = __expf(G[2 * e + 1]);
                const float ia = __expf(-G[2 * e]), ib = __expf(-G[2 * e + 1]);
                const float ka = fk * bf16_lo(kw[e]), kb = fk * bf16_hi(kw[e]);
                const float qa = fq * bf16_lo(qw[e]), qb = fq * bf16_hi(qw[e]);
                kt[e] = pack_bf16x2(ka * ea, kb * eb);
                qt[e] = pack_bf16x2(qa * ea, qb * eb);
                kh[e] = pack_bf16x2(ka * ia, kb * ib);
                kcw[e] = pack_bf16x2(ka * (egc[c0 + 2 * e] * ia), kb * (egc[c0 + 2 * e + 1] * ib));
            }
            *reinterpret_cast<uint4 *>(sm + okt) = make_uint4(kt[0], kt[1], kt[2], kt[3]);
            *reinterpret_cast<uint4 *>(sm + oqt) = make_uint4(qt[0], qt[1], qt[2], qt[3]);
            *reinterpret_cast<uint4 *>(sm + A_KH + o) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
            *reinterpret_cast<uint4 *>(kc + o) = make_uint4(kcw[0], kcw[1], kcw[2], kcw[3]);
        }
    }
    fence_proxy_async_smem();  // the tiles are read by the tensor cores and the bulk copies
    __syncthreads();

    // ---- [A_raw; P] = [Kt; Qt] Kh^T: one M = 128, N = 64, K = 128 product into TMEM columns
    //      0-63 (lanes 0-63 the rows of Kt Kh^T, lanes 64-127 those of Qt Kh^T); Qt -> record
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(sb + A_KQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sb + A_KH + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
            umma_bf16(tmem, ad, bd, ID_AP, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_mma);
        bulk_store(rec + REC_QT, sb + A_KQ + 8192, 8192);
        bulk_store(rec + REC_QT + 8192, sb + A_KQ + 16384 + 8192, 8192);
        bulk_commit_group();
    }
    if (__syncthreads_or(!mbar_wait_bounded(bar_mma, 0))) {
        abort_cta(bar_mma, 0);
        return;
    }
    tc_fence_after();
    {
        // warp w reads TMEM lanes 32 (w & 3) .. +31 (one row each), columns 32 (w >> 2) .. +31
        const int quad = warp & 3, s0 = 32 * (warp >> 2);
        uint32_t d[32];
        tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + s0, d);
        tmem_wait_ld();
        if (quad < 2) {  // A_rs = beta_r (Kt Kh^T)_rs, s < r, fp32 for the solve
            const int r = 32 * quad + lane;
            const float br = r < n ? sbeta[r] : 0.f;
            float *arow = As + r * AS_LD + s0;
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
                float v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    v[e] = (s0 + 4 * j4 + e < r) ? br * __uint_as_float(d[4 * j4 + e]) : 0.f;
                *reinterpret_cast<float4 *>(arow + 4 * j4) = make_float4(v[0], v[1], v[2], v[3]);
            }
        } else {  // P_rs = (Qt Kh^T)_rs, s <= r, bf16 into the (now free) Kh slot
            const int r = 32 * (quad - 2) + lane;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int s = s0 + 8 * u + 2 * e;
                    w[e] = pack_bf16x2((s <= r && r < n) ? __uint_as_float(d[8 * u + 2 * e]) : 0.f,
                                       (s + 1 <= r && r < n) ? __uint_as_float(d[8 * u + 2 * e + 1]) : 0.f);
                }
                *reinterpret_cast<uint4 *>(sm + A_KH + toff(r, s0 + 8 * u, 64)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        if (tid < kD) reinterpret_cast<float *>(sm + A_KH + 8192)[tid] = egc[tid];
    }
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {  // P and e^{G_C} (contiguous in the record) -> record
        bulk_store(rec + REC_P, sb + A_KH, 8192 + 512);
        bulk_commit_group();
    }

    // ---- X = (I + A)^-1 (16x16 blocks, fp32) and, as its blocks appear, T = X Diag(beta)
    //      (bf16 [r][s], the K-major B operand below) in the Qt slot, free once Qt's bulk store
    //      has read it ------------------------------------------------------------------------
    if (tid == 0) bulk_wait_group_read<1>();  // the Qt group; the P group may still be reading
    __syncthreads();
    uint8_t *Tt = sm + A_T;
    if (tid < 64) {  // diagonal blocks by forward substitution, one column per thread
        const int bi = tid >> 4, c0 = tid & 15;
        const float *ab = As + bi * 16 * AS_LD + bi * 16;
        const float bc = sbeta[bi * 16 + c0];
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < r; ++s2) acc += ab[r * AS_LD + s2] * x[s2];
            x[r] = r < c0 ? 0.f : (r == c0 ? 1.f : -acc);
            Xs[(bi * 16 + r) * AS_LD + bi * 16 + c0] = x[r];
            *reinterpret_cast<__nv_bfloat16 *>(Tt + toff(bi * 16 + r, bi * 16 + c0, 64)) =
                __float2bfloat16_rn(x[r] * bc);
        }
    } else {  // the blocks above the diagonal of T are zero: 6 blocks x 16 rows x 32 bytes
        for (int idx = tid - 64; idx < 6 * 16 * 2; idx += NT - 64) {
            const int blk = idx >> 5, rr = (idx >> 1) & 15, hh = idx & 1;
            const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);           // block row
            const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);  // block column > bi
            *reinterpret_cast<uint4 *>(Tt + toff(bi * 16 + rr, bj * 16 + hh * 8, 64)) =
                make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    solve_level<1>(As, Xs, Ys, tid, Tt, sbeta);
    solve_level<2>(As, Xs, Ys, tid, Tt, sbeta);
    solve_level<3>(As, Xs, Ys, tid, Tt, sbeta);
    fence_proxy_async_smem();  // T is read by the tensor cores
    __syncthreads();

    // ---- W^T = Kt^T T^T and Ut^T = V^T T^T: M = 128 (d), N = 64 (r), K = 64 (s), with Kt and V
    //      read MN-major; W^T into TMEM columns 64-127, Ut^T into columns 0-63 -----------------
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(sb + A_T + kk * 32, 16, 1024);
            const uint64_t aw = smem_desc_sw128(sb + A_KQ + kk * 2048, 16384, 1024);
            const uint64_t au = smem_desc_sw128(sb + A_V + kk * 2048, 8192, 1024);
            umma_bf16(tmem + 64, aw, bd, ID_WU, kk > 0 ? 1u : 0u);
            umma_bf16(tmem, au, bd, ID_WU, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_mma);
    }
    if (__syncthreads_or(!mbar_wait_bounded(bar_mma, 1))) {
        abort_cta(bar_mma, 1);
        return;
    }
    tc_fence_after();
    {
        // thread row dd of d_k (warps 0-3: -W^T, into the free V slot) or of d_v (warps 4-7:
        // Ut^T); 32 token columns per TMEM load, stored as four 16-byte chunks of the row
        const int quad = warp & 3, dd = 32 * quad + lane;
        const bool w_side = warp < 4;
        const float sgn = w_side ? -1.f : 1.f;
        uint8_t *dst = sm + (w_side ? A_V : A_UT);
        uint32_t d[32];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + (w_side ? 64 : 0) + 32 * hr, d);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w[e] = pack_bf16x2(sgn * __uint_as_float(d[8 * u + 2 * e]),
                                       sgn * __uint_as_float(d[8 * u + 2 * e + 1]));
                *reinterpret_cast<uint4 *>(dst + toff(dd, 32 * hr + 8 * u, 128)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        bulk_store(rec + REC_NW, sb + A_V, 16384);
        bulk_store(rec + REC_UT, sb + A_UT, 16384);
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
// Per chunk c (p = c & 1 picks the stage, the M buffer and the U buffer):
//   phase 1  bf16 copy of M -> M[p]; st <- e^{G_C} st                 | barrier; issue chunk c+1
//   phase 2  U = Ut - W M and O = Qt M, sharing M's fragments; U -> U[p] | barrier
//   phase 3  O += P U, store O; st += Kc^T U
// Two barriers per chunk: the buffers a chunk writes were last read two phases earlier.
__global__ void __launch_bounds__(kThreads, 1) prefill_scan_kernel(const PrefillScanArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + B_BAR);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int l7 = lane & 7, lb3 = (lane >> 3) & 1, lb4 = lane >> 4;
    const int bh = blockIdx.x / kSplitV, sv = blockIdx.x - bh * kSplitV;
    const int b = bh / a.H, h = bh - b * a.H;
    const int col0 = sv * kDV;  // this CTA's first d_v column
    const int T = a.T;
    griddep_launch_dependents();
    griddep_wait();  // the records are the prep pass's output
    const int slot = a.slots ? a.slots[b] : b;
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) atomicOr(&g_err, HMD_DEVERR_SLOT);
        return;
    }
    float *Mg = a.state + ((size_t)slot * a.H + h) * kD * kD;
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o);

    if (tid == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        fence_barrier_init();
    }
    __syncthreads();
    auto issue = [&](int c) {  // thread 0: chunk c's record head -> stage c & 1
        const uint32_t bar = smem_u32(&bars[c & 1]);
        mbar_arrive_expect_tx(bar, REC_BYTES);
        bulk_load(sb + (c & 1) * B_STAGE, record(a, bh, c), REC_BYTES, bar);
    };
    if (tid == 0) issue(0);

    // state strip of this warp: rows 16*warp + g (+8), slice columns 8*nt + 2*t4 (+1)
    const int sr0 = 16 * warp + g, sr1 = sr0 + 8;
    float st[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int cc = col0 + nt * 8 + 2 * t4;
        const float2 x0 = *reinterpret_cast<const float2 *>(Mg + (size_t)sr0 * kD + cc);
        const float2 x1 = *reinterpret_cast<const float2 *>(Mg + (size_t)sr1 * kD + cc);
        st[nt][0] = x0.x; st[nt][1] = x0.y; st[nt][2] = x1.x; st[nt][3] = x1.y;
    }
    // U / O role: chunk rows 16*rt + g (+8), slice columns 32*chh + 8*j + 2*t4 (+1)
    const int rt = warp & 3, chh = warp >> 2;
    const int ur0 = 16 * rt + g, ur1 = ur0 + 8;

    int aborted_at = -1;
    for (int c = 0; c < a.n_seg; ++c) {
        const int p = c & 1;
        const uint32_t stg = sb + p * B_STAGE;
        const uint32_t mb = sb + B_M + p * 16384, ub = sb + B_U + p * 8192;
        const int t0 = (a.chunk_begin + c) * kC;
        const int n = min(kC, T - t0);
        const bool ok = mbar_wait_bounded(smem_u32(&bars[p]), (c >> 1) & 1);
        // ---- phase 1: bf16 copy of M (the B operand of U and O); st <- e^{G_C} st ---------
        if (ok) {
            const float *gm = reinterpret_cast<const float *>(sm + p * B_STAGE + REC_GAM);
            const float g0 = gm[sr0], g1 = gm[sr1];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int cc = nt * 8 + 2 * t4;
                st_bf16x2(sm + B_M + p * 16384, toff(sr0, cc, 128), st[nt][0], st[nt][1]);
                st_bf16x2(sm + B_M + p * 16384, toff(sr1, cc, 128), st[nt][2], st[nt][3]);
                st[nt][0] *= g0; st[nt][1] *= g0; st[nt][2] *= g1; st[nt][3] *= g1;
            }
        }
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
            aborted_at = c;
            break;
        }
        if (tid == 0 && c + 1 < a.n_seg) {  // every warp is past chunk c-1: its stage is free
            fence_proxy_async_smem();
            issue(c + 1);
        }

        // ---- phase 2: U = Ut + (-W) M and O = Qt M (16 rows x 32 columns per warp) -------
        float u[4][4], o[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // Ut[token][cc], Ut[token][cc + 1] from rows cc, cc + 1 of the stage's Ut^T tile
            const int cc = col0 + 32 * chh + 8 * j + 2 * t4;
            const uint8_t *ut = sm + p * B_STAGE + REC_UT;
            u[j][0] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(ut + toff(cc, ur0, 128)));
            u[j][1] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(ut + toff(cc + 1, ur0, 128)));
            u[j][2] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(ut + toff(cc, ur1, 128)));
            u[j][3] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(ut + toff(cc + 1, ur1, 128)));
#pragma unroll
            for (int e = 0; e < 4; ++e) o[j][e] = 0.f;
        }
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
            uint32_t aw[4], aq[4];
            ldmatrix_x4_trans(stg + REC_NW + toff(kk * 16 + l7 + lb4 * 8, 16 * rt + lb3 * 8, 128),
                              aw[0], aw[1], aw[2], aw[3]);
            ldmatrix_x4(stg + REC_QT + toff(16 * rt + l7 + lb3 * 8, kk * 16 + lb4 * 8, 64), aq[0], aq[1],
                        aq[2], aq[3]);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(mb + toff(kk * 16 + l7 + lb3 * 8, 32 * chh + np * 16 + lb4 * 8, 128),
                                  b0, b1, b2, b3);
                mma_bf16_16816(u[2 * np], aw, b0, b1);
                mma_bf16_16816(u[2 * np + 1], aw, b2, b3);
                mma_bf16_16816(o[2 * np], aq, b0, b1);
                mma_bf16_16816(o[2 * np + 1], aq, b2, b3);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int cc = 32 * chh + 8 * j + 2 * t4;
            st_bf16x2(sm + B_U + p * 8192, toff(ur0, cc, 64), u[j][0], u[j][1]);
            st_bf16x2(sm + B_U + p * 8192, toff(ur1, cc, 64), u[j][2], u[j][3]);
        }
        __syncthreads();

        // ---- phase 3: O += P U and store it; st += Kc^T U ------------------------------------
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk) {
            uint32_t af[4];
            ldmatrix_x4(stg + REC_P + toff(16 * rt + l7 + lb3 * 8, kk * 16 + lb4 * 8, 64), af[0],
                        af[1], af[2], af[3]);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(ub + toff(kk * 16 + l7 + lb3 * 8, 32 * chh + np * 16 + lb4 * 8, 64),
                                  b0, b1, b2, b3);
                mma_bf16_16816(o[2 * np], af, b0, b1);
                mma_bf16_16816(o[2 * np + 1], af, b2, b3);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int cc = col0 + 32 * chh + 8 * j + 2 * t4;
            if (ur0 < n)
                *reinterpret_cast<uint32_t *>(og + (((size_t)b * T + t0 + ur0) * a.H + h) * kD + cc) =
                    pack_bf16x2(a.scale * o[j][0], a.scale * o[j][1]);
            if (ur1 < n)
                *reinterpret_cast<uint32_t *>(og + (((size_t)b * T + t0 + ur1) * a.H + h) * kD + cc) =
                    pack_bf16x2(a.scale * o[j][2], a.scale * o[j][3]);
        }
        // st += Kc^T U (this warp's 16 rows of d_k, all 64 slice columns)
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk) {
            uint32_t af[4];
            ldmatrix_x4_trans(stg + REC_KC + toff(kk * 16 + l7 + lb4 * 8, 16 * warp + lb3 * 8, 64), af[0],
                              af[1], af[2], af[3]);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(ub + toff(kk * 16 + l7 + lb3 * 8, np * 16 + lb4 * 8, 64), b0, b1, b2, b3);
                mma_bf16_16816(st[2 * np], af, b0, b1);
                mma_bf16_16816(st[2 * np + 1], af, b2, b3);
            }
        }
    }
    if (aborted_at >= 0) {
        // a wait gave up: let this CTA's one bulk copy in flight (chunk aborted_at) finish,
        // bounded; the state is left as it was at the start of this segment
        if (tid == 0)
            (void)mbar_wait_bounded(smem_u32(&bars[aborted_at & 1]), (aborted_at >> 1) & 1);
        return;
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int cc = col0 + nt * 8 + 2 * t4;
        *reinterpret_cast<float2 *>(Mg + (size_t)sr0 * kD + cc) = make_float2(st[nt][0], st[nt][1]);
        *reinterpret_cast<float2 *>(Mg + (size_t)sr1 * kD + cc) = make_float2(st[nt][2], st[nt][3]);
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
        cudaError_t e = cudaFuncSetAttribute(prefill_prep_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)A_SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_prep_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)A_SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)B_SMEM);
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
                            32, false))
            return cudaErrorInvalidValue;
    } else {
        tmg = tmq;  // not read
    }
    PrefillScanArgs p;
    p.q = a.q; p.k = a.k; p.v = a.v; p.beta = a.beta; p.log_gate = a.log_gate;
    p.state = a.state; p.slots = a.slots; p.n_slots = a.n_slots; p.o = a.o;
    p.B = a.B; p.T = a.T; p.H = a.H; p.scale = a.scale; p.ws = ws; p.act = a.act;
    for (int cb = 0; cb < n_chunks; cb += seg) {
        p.chunk_begin = cb;
        p.n_seg = std::min(seg, n_chunks - cb);
        const unsigned grid_a = (unsigned)(bhs * p.n_seg);
        cudaError_t e = launch_pdl(a.kind == HMD_KDA ? prefill_prep_kernel<true> : prefill_prep_kernel<false>,
                                   dim3(grid_a), dim3(kPrepThreads), A_SMEM, s, tmq, tmk, tmv, tmg, p);
        if (e != cudaSuccess) return e;
        e = launch_pdl(prefill_scan_kernel, dim3((unsigned)(bhs * kSplitV)), dim3(kThreads), B_SMEM, s,
                       p);
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

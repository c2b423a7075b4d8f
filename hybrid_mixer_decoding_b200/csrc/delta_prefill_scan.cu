// Chunked delta-rule prefill in two passes on tensor cores (mma.sync m16n8k16, bf16 operands,
// fp32 accumulation), bf16 activations, d_k = d_v = 128, chunk C = 64.
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
// Pass A (prefill_prep_kernel): one CTA per (sequence, head, chunk), all chunks at once. It
// computes the gate factors, A and P, the blocked UT solve, W and Ut, and writes one record per
// chunk: Qt, -W, Kc, P (bf16, already in the 128-byte XOR-swizzled tile layout pass B reads with
// ldmatrix), e^{G_C} and Ut^T (fp32, rows of d_v).
// Pass B (prefill_scan_kernel): one CTA per (sequence, head, half of d_v) walks the chunks in
// order. Each chunk's record arrives by one bulk copy into a 2-stage shared-memory ring while
// the chunk before it computes; the state half lives in registers as MMA accumulator fragments.
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
constexpr uint32_t REC_NW = 16384;     // -W  bf16 [64][128]
constexpr uint32_t REC_KC = 32768;     // Kc  bf16 [64][128]
constexpr uint32_t REC_P = 49152;      // P   bf16 [64][64]
constexpr uint32_t REC_GAM = 57344;    // e^{G_C} fp32 [128]
constexpr uint32_t REC_HEAD = 57856;   // bytes above, moved by one bulk copy
constexpr uint32_t REC_UT = 57856;     // Ut^T fp32 [128 d_v][64 tokens] (see utt_idx)
constexpr uint32_t REC_BYTES = REC_UT + kC * kD * 4;  // 90624
static_assert(REC_HEAD % 16 == 0 && REC_BYTES % 16 == 0, "bulk copies need 16-byte sizes");

// ---- pass A shared memory (bytes from a 1024-aligned base) ---------------------------------
constexpr uint32_t A_KT = 0;           // Kt [64][128]; at the end -W (bf16, record layout)
constexpr uint32_t A_QT = 16384;       // q, then Qt [64][128]
constexpr uint32_t A_KH = 32768;       // k, then Kh [64][128]; then P + e^{G_C}; at the end
constexpr uint32_t A_V = 49152;        //   Ut fp32 across Kh and V (32 KiB, record layout)
constexpr uint32_t A_G = 65536;        // KDA log-gates -> in-chunk prefix, fp32 [64][128]
constexpr uint32_t A_AS = 65536;       // after the gate pass: A fp32 [64][68], then T bf16
constexpr uint32_t A_XS = 82944;       // X fp32 [64][68]
constexpr uint32_t A_YS = 100352;      // Y fp32 [3][16][20]
constexpr uint32_t A_SMALL = 104192;
constexpr uint32_t A_SMEM = A_SMALL + 3584 + 1024;
constexpr uint32_t A_T = A_AS;
constexpr int AS_LD = 68;
constexpr int YS_LD = 20;
static_assert(A_G + kC * kD * 4 <= A_YS, "log-gate staging fits the A/X region");

// ---- pass B shared memory ----------------------------------------------------------------
constexpr uint32_t B_STAGE = 58368;        // one record head, padded to 1 KiB
constexpr uint32_t B_M = 2 * B_STAGE;      // M bf16 [128][64], two buffers (chunk parity)
constexpr uint32_t B_U = B_M + 2 * 16384;  // U bf16 [64][64], two buffers
constexpr uint32_t B_BAR = B_U + 2 * 8192;
constexpr uint32_t B_SMEM = B_BAR + 64 + 1024;

// byte offset of element (row, col) of a tile whose halves (64 columns each) hold `rows` rows
__device__ __forceinline__ uint32_t toff(int row, int col, int rows) {
    return (uint32_t)((col >> 6) * rows * 128 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                      ((col & 7) << 1));
}

// word index of Ut[token][dv] in the Ut^T block: rows of 64 tokens per d_v column, the 8-word
// groups XOR-permuted by row so that a warp's fragment stores hit distinct banks
__device__ __forceinline__ int utt_idx(int dv, int tok) { return dv * kC + (tok ^ ((dv & 7) << 3)); }

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
__device__ __forceinline__ void solve_level(const float *As, float *Xs, float *Ys, int tid) {
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
        if (part == 0)
            *reinterpret_cast<float4 *>(Xs + (i * 16 + r) * AS_LD + j * 16 + cg * 4) =
                make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    __syncthreads();
}

template <bool KDA>
__global__ void __launch_bounds__(kPrepThreads, 2) prefill_prep_kernel(const PrefillScanArgs a) {
    constexpr int NT = kPrepThreads;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    float *Gs = reinterpret_cast<float *>(sm + A_G);
    float *As = reinterpret_cast<float *>(sm + A_AS);
    float *Xs = reinterpret_cast<float *>(sm + A_XS);
    float *Ys = reinterpret_cast<float *>(sm + A_YS);
    float *sbeta = reinterpret_cast<float *>(sm + A_SMALL);  // [64]
    float *qoff = sbeta + 64;                                 // [NQ][128] KDA: gate sums of
                                                              //   the row parts, then their
                                                              //   exclusive prefix
    float *lgp = qoff + 512;                                  // [64] GDN log-gate prefix
    float *wsum = lgp + 64;                                   // [2]
    float *egc = wsum + 2;                                    // [128] e^{G_C}

    constexpr int NQ = NT / kD;       // KDA gate prefix: row parts per channel
    constexpr int RPQ = kC / NQ;      // rows per part
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int l7 = lane & 7, lb3 = (lane >> 3) & 1, lb4 = lane >> 4;
    const int bh = blockIdx.x / a.n_seg, c = blockIdx.x - bh * a.n_seg;
    const int b = bh / a.H, h = bh - b * a.H;
    const int T = a.T;
    const int t0 = (a.chunk_begin + c) * kC;
    const int n = min(kC, T - t0);
    uint8_t *rec = record(a, bh, c);
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q);
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(a.k);
    const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(a.v);
    griddep_launch_dependents();
    griddep_wait();  // the inputs may come from the previous kernel

    // ---- stage q (into the Qt slot), k (into the Kh slot), v, KDA log-gates; beta ----------
    {
        constexpr int J16 = kC * kD / 8 / NT;  // 16-byte pieces of a bf16 tile per thread
        constexpr int JG = kC * kD / 4 / NT;   // float4 pieces of the KDA gate tile per thread
        const size_t row0 = ((size_t)b * T + t0) * a.H + h;  // token t0's row in [B][T][H]
        uint4 qv[J16], kv[J16], vv[J16];
#pragma unroll
        for (int j = 0; j < J16; ++j) {
            const int idx = tid + j * NT, r = idx >> 4, ch = idx & 15;
            qv[j] = kv[j] = vv[j] = make_uint4(0, 0, 0, 0);
            if (r < n) {
                const size_t off = (row0 + (size_t)r * a.H) * kD + ch * 8;
                qv[j] = __ldg(reinterpret_cast<const uint4 *>(qg + off));
                kv[j] = __ldg(reinterpret_cast<const uint4 *>(kg + off));
                vv[j] = __ldg(reinterpret_cast<const uint4 *>(vg + off));
            }
        }
        float4 gv[JG];
        if constexpr (KDA) {
#pragma unroll
            for (int j = 0; j < JG; ++j) {
                const int idx = tid + j * NT, r = idx >> 5, c4 = idx & 31;
                gv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (r < n)
                    gv[j] = __ldg(reinterpret_cast<const float4 *>(a.log_gate + (row0 + (size_t)r * a.H) * kD + c4 * 4));
            }
        }
#pragma unroll
        for (int j = 0; j < J16; ++j) {
            const int idx = tid + j * NT, r = idx >> 4, ch = idx & 15;
            const uint32_t o = toff(r, ch * 8, 64);
            *reinterpret_cast<uint4 *>(sm + A_QT + o) = qv[j];
            *reinterpret_cast<uint4 *>(sm + A_KH + o) = kv[j];
            *reinterpret_cast<uint4 *>(sm + A_V + o) = vv[j];
        }
        if constexpr (KDA) {
#pragma unroll
            for (int j = 0; j < JG; ++j) {
                const int idx = tid + j * NT, r = idx >> 5, c4 = idx & 31;
                *reinterpret_cast<float4 *>(Gs + r * kD + c4 * 4) = gv[j];
            }
        }
        if (tid < kC) {
            const size_t tok = row0 + (size_t)tid * a.H;
            sbeta[tid] = tid < n ? a.beta[tok] : 0.f;
            if constexpr (!KDA) {
                float x = tid < n ? a.log_gate[tok] : 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, off);
                    if (lane >= off) x += y;
                }
                if (lane == 31) wsum[warp] = x;
                lgp[tid] = x;
            }
        }
    }
    __syncthreads();

    // ---- gate prefix G (log domain): KDA per channel in place within NQ row parts, plus the
    //      parts' exclusive prefix; GDN per token -------------------------------------------------
    if constexpr (KDA) {
        const int i = tid & (kD - 1), qr = tid >> 7;
        float run = 0.f;
#pragma unroll
        for (int r = RPQ * qr; r < RPQ * qr + RPQ; ++r) {
            run += Gs[r * kD + i];
            Gs[r * kD + i] = run;
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
        }
    } else {
        if (tid < kC) lgp[tid] += (warp == 1 ? wsum[0] : 0.f);
        __syncthreads();
        if (tid < kD) egc[tid] = __expf(lgp[kC - 1]);
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
            const uint4 qr = *reinterpret_cast<const uint4 *>(sm + A_QT + o);
            const uint4 kr = *reinterpret_cast<const uint4 *>(sm + A_KH + o);
            float G[8];
            if constexpr (KDA) {
                const float4 g0 = *reinterpret_cast<const float4 *>(Gs + r * kD + c0);
                const float4 g1 = *reinterpret_cast<const float4 *>(Gs + r * kD + c0 + 4);
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
            uint32_t kt[4], qt[4], kh[4], kcw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float ea = __expf(G[2 * e]), eb = __expf(G[2 * e + 1]);
                const float ia = __expf(-G[2 * e]), ib = __expf(-G[2 * e + 1]);
                const float ka = bf16_lo(kw[e]), kb = bf16_hi(kw[e]);
                const float qa = bf16_lo(qw[e]), qb = bf16_hi(qw[e]);
                kt[e] = pack_bf16x2(ka * ea, kb * eb);
                qt[e] = pack_bf16x2(qa * ea, qb * eb);
                kh[e] = pack_bf16x2(ka * ia, kb * ib);
                kcw[e] = pack_bf16x2(ka * (egc[c0 + 2 * e] * ia), kb * (egc[c0 + 2 * e + 1] * ib));
            }
            *reinterpret_cast<uint4 *>(sm + A_KT + o) = make_uint4(kt[0], kt[1], kt[2], kt[3]);
            *reinterpret_cast<uint4 *>(sm + A_QT + o) = make_uint4(qt[0], qt[1], qt[2], qt[3]);
            *reinterpret_cast<uint4 *>(sm + A_KH + o) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
            *reinterpret_cast<uint4 *>(kc + o) = make_uint4(kcw[0], kcw[1], kcw[2], kcw[3]);
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {  // Qt -> record
        bulk_store(rec + REC_QT, sb + A_QT, 16384);
        bulk_commit_group();
    }

    // ---- A and P: [Kt | Qt] Kh^T; each warp 16 rows x (64 / NH) columns -------------------
    {
        constexpr int NH = NT / 256;  // warps per 16-row strip of A or P
        constexpr int NP = 4 / NH;    // 16-column pairs per warp (n-tiles = 2 NP)
        const int mat = warp / (4 * NH), rt = (warp / NH) & 3, nh = warp % NH;
        const uint32_t abase = sb + (mat ? A_QT : A_KT);
        float acc[2 * NP][4];
#pragma unroll
        for (int i = 0; i < 2 * NP; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
            uint32_t af[4];
            ldmatrix_x4(abase + toff(16 * rt + l7 + lb3 * 8, kk * 16 + lb4 * 8, 64), af[0], af[1],
                        af[2], af[3]);
#pragma unroll
            for (int np = 0; np < NP; ++np) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(sb + A_KH + toff(16 * NP * nh + np * 16 + l7 + lb4 * 8, kk * 16 + lb3 * 8, 64),
                            b0, b1, b2, b3);
                mma_bf16_16816(acc[2 * np], af, b0, b1);
                mma_bf16_16816(acc[2 * np + 1], af, b2, b3);
            }
        }
        __syncthreads();  // Kh is read by every warp above; P and e^{G_C} take its place below
        const int r0 = 16 * rt + g, r1 = r0 + 8;
#pragma unroll
        for (int nt = 0; nt < 2 * NP; ++nt) {
            const int s0 = 16 * NP * nh + nt * 8 + 2 * t4;
            if (mat == 0) {
                As[r0 * AS_LD + s0] = (s0 < r0 && r0 < n) ? sbeta[r0] * acc[nt][0] : 0.f;
                As[r0 * AS_LD + s0 + 1] = (s0 + 1 < r0 && r0 < n) ? sbeta[r0] * acc[nt][1] : 0.f;
                As[r1 * AS_LD + s0] = (s0 < r1 && r1 < n) ? sbeta[r1] * acc[nt][2] : 0.f;
                As[r1 * AS_LD + s0 + 1] = (s0 + 1 < r1 && r1 < n) ? sbeta[r1] * acc[nt][3] : 0.f;
            } else {
                st_bf16x2(sm + A_KH, toff(r0, s0, 64), (s0 <= r0 && r0 < n) ? acc[nt][0] : 0.f,
                          (s0 + 1 <= r0 && r0 < n) ? acc[nt][1] : 0.f);
                st_bf16x2(sm + A_KH, toff(r1, s0, 64), (s0 <= r1 && r1 < n) ? acc[nt][2] : 0.f,
                          (s0 + 1 <= r1 && r1 < n) ? acc[nt][3] : 0.f);
            }
        }
        if (tid < kD) reinterpret_cast<float *>(sm + A_KH + 8192)[tid] = egc[tid];
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {  // P and e^{G_C} (contiguous in the record) -> record
        bulk_store(rec + REC_P, sb + A_KH, 8192 + 512);
        bulk_commit_group();
    }

    // ---- X = (I + A)^-1 (16x16 blocks, fp32), T = X Diag(beta) ----------------------------
    if (tid < 64) {  // diagonal blocks by forward substitution, one column per thread
        const int bi = tid >> 4, c0 = tid & 15;
        const float *ab = As + bi * 16 * AS_LD + bi * 16;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < r; ++s2) acc += ab[r * AS_LD + s2] * x[s2];
            x[r] = r < c0 ? 0.f : (r == c0 ? 1.f : -acc);
            Xs[(bi * 16 + r) * AS_LD + bi * 16 + c0] = x[r];
        }
    }
    __syncthreads();
    solve_level<1>(As, Xs, Ys, tid);
    solve_level<2>(As, Xs, Ys, tid);
    solve_level<3>(As, Xs, Ys, tid);
    // T overwrites A (no longer read)
    for (int idx = tid; idx < 64 * 32; idx += NT) {
        const int r = idx >> 5, s0 = (idx & 31) * 2;
        const float v0 = s0 <= r ? Xs[r * AS_LD + s0] * sbeta[s0] : 0.f;
        const float v1 = s0 + 1 <= r ? Xs[r * AS_LD + s0 + 1] * sbeta[s0 + 1] : 0.f;
        st_bf16x2(sm + A_T, toff(r, s0, 64), v0, v1);
    }
    __syncthreads();

    // ---- W = T Kt (warps 4-7, 16 token rows x 128 each) and Ut^T = V^T T^T (warps 0-3,
    //      32 d_v rows x 64 tokens each) ---------------------------------------------------
    {
        static_assert(NT == 256, "one warp per 16 rows of W, per 32 rows of Ut^T");
        const int rt = warp & 3;
        float acc[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
        if (warp >= 4) {
#pragma unroll
            for (int kk = 0; kk < kC / 16; ++kk) {
                uint32_t af[4];
                ldmatrix_x4(sb + A_T + toff(16 * rt + l7 + lb3 * 8, kk * 16 + lb4 * 8, 64), af[0], af[1],
                            af[2], af[3]);
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(sb + A_KT + toff(kk * 16 + l7 + lb3 * 8, np * 16 + lb4 * 8, 64),
                                      b0, b1, b2, b3);
                    mma_bf16_16816(acc[2 * np], af, b0, b1);
                    mma_bf16_16816(acc[2 * np + 1], af, b2, b3);
                }
            }
        } else {
            // A = V^T (rows d_v) by transposed loads of V [token][d_v]; B = T^T from T [r][s]
#pragma unroll
            for (int kk = 0; kk < kC / 16; ++kk) {
                uint32_t af[2][4];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
                    ldmatrix_x4_trans(sb + A_V + toff(kk * 16 + l7 + lb4 * 8, 32 * rt + 16 * mt + lb3 * 8, 64),
                                      af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(sb + A_T + toff(np * 16 + lb4 * 8 + l7, kk * 16 + lb3 * 8, 64), b0, b1,
                                b2, b3);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        mma_bf16_16816(acc[8 * mt + 2 * np], af[mt], b0, b1);
                        mma_bf16_16816(acc[8 * mt + 2 * np + 1], af[mt], b2, b3);
                    }
                }
            }
        }
        if (tid == 0) bulk_wait_group_read0();  // P's bulk store has left the Kh region
        __syncthreads();  // Kt and V are no longer read: -W and Ut^T take their place
        if (warp >= 4) {
            const int r0 = 16 * rt + g, r1 = r0 + 8;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                const int cc = nt * 8 + 2 * t4;
                st_bf16x2(sm + A_KT, toff(r0, cc, 64), -acc[nt][0], -acc[nt][1]);
                st_bf16x2(sm + A_KT, toff(r1, cc, 64), -acc[nt][2], -acc[nt][3]);
            }
        } else {
            float *ut = reinterpret_cast<float *>(sm + A_KH);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int d0 = 32 * rt + 16 * mt + g, d1 = d0 + 8;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    const int tk = nt * 8 + 2 * t4;
                    *reinterpret_cast<float2 *>(ut + utt_idx(d0, tk)) =
                        make_float2(acc[8 * mt + nt][0], acc[8 * mt + nt][1]);
                    *reinterpret_cast<float2 *>(ut + utt_idx(d1, tk)) =
                        make_float2(acc[8 * mt + nt][2], acc[8 * mt + nt][3]);
                }
            }
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        bulk_store(rec + REC_NW, sb + A_KT, 16384);
        bulk_store(rec + REC_UT, sb + A_KH, 32768);
        bulk_commit_group();
        bulk_wait_group_read0();  // shared memory must outlive the copies' reads
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
        mbar_arrive_expect_tx(bar, REC_HEAD);
        bulk_load(sb + (c & 1) * B_STAGE, record(a, bh, c), REC_HEAD, bar);
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
    float un[4][4];  // Ut of the next chunk, prefetched
    auto load_ut = [&](int c) {
        const float *ut = reinterpret_cast<const float *>(record(a, bh, c) + REC_UT);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int cc = col0 + 32 * chh + 8 * j + 2 * t4;
            un[j][0] = ut[utt_idx(cc, ur0)];
            un[j][1] = ut[utt_idx(cc + 1, ur0)];
            un[j][2] = ut[utt_idx(cc, ur1)];
            un[j][3] = ut[utt_idx(cc + 1, ur1)];
        }
    };
    load_ut(0);

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
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                u[j][e] = un[j][e];
                o[j][e] = 0.f;
            }
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
            uint32_t aw[4], aq[4];
            ldmatrix_x4(stg + REC_NW + toff(16 * rt + l7 + lb3 * 8, kk * 16 + lb4 * 8, 64), aw[0], aw[1],
                        aw[2], aw[3]);
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
        if (c + 1 < a.n_seg) load_ut(c + 1);
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
    static cudaError_t attr = [] {
        cudaError_t e = cudaFuncSetAttribute(prefill_prep_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)A_SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_prep_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)A_SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)B_SMEM);
        return e;
    }();
    if (attr != cudaSuccess) return attr;
    const long long bhs = (long long)a.B * a.H;
    const int n_chunks = (a.T + kC - 1) / kC;
    if (bhs <= 0 || n_chunks <= 0) return cudaSuccess;
    const long long fit = (long long)(ws_bytes / ((size_t)bhs * REC_BYTES));
    if (fit < 1 || (reinterpret_cast<uintptr_t>(ws) & 15)) return cudaErrorInvalidValue;
    const int seg = (int)std::min<long long>(n_chunks, fit);
    PrefillScanArgs p;
    p.q = a.q; p.k = a.k; p.v = a.v; p.beta = a.beta; p.log_gate = a.log_gate;
    p.state = a.state; p.slots = a.slots; p.n_slots = a.n_slots; p.o = a.o;
    p.B = a.B; p.T = a.T; p.H = a.H; p.scale = a.scale; p.ws = ws;
    for (int cb = 0; cb < n_chunks; cb += seg) {
        p.chunk_begin = cb;
        p.n_seg = std::min(seg, n_chunks - cb);
        const unsigned grid_a = (unsigned)(bhs * p.n_seg);
        cudaError_t e = launch_pdl(a.kind == HMD_KDA ? prefill_prep_kernel<true> : prefill_prep_kernel<false>,
                                   dim3(grid_a), dim3(kPrepThreads), A_SMEM, s, p);
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

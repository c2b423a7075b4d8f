// Chunked delta-rule prefill on tensor cores (mma.sync m16n8k16, bf16 in / fp32 accumulate),
// bf16 activations, d_k = d_v = 128, chunk C = 64.
//
// Same chunk algebra as delta_prefill.cu (the standard WY / UT-transform rewriting of the gated
// delta rule for the GDN and KDA mixers of "Super Apriel: One Checkpoint, Many Speeds",
// abstract; gist.science technical summary, section 2a). Per chunk, with the state M ([d_k][d_v],
// fp32) at the chunk start and G the per-channel cumulative log-gate:
//   Kt = k e^G, Kh = k e^-G, Qt = q e^G                              (gate pass, CUDA cores)
//   A = beta_r (Kt Kh^T)_{rs} (s < r),  P = (Qt Kh^T)_{rs} (s <= r)   (tensor cores)
//   T = (I + A)^-1 Diag(beta)                                          (16x16-blocked, fp32)
//   W = T Kt,  Ut = T V                                                (tensor cores)
//   U = Ut - W M,  O = Qt M + P U                                      (tensor cores)
//   M_next = Diag(e^{G_C}) (M + Kh^T U)                                (tensor cores)
// One CTA of 8 warps per (sequence, head) runs the chunks in order. The fp32 state lives in
// registers as accumulator fragments (warp w owns rows 16w..16w+15), so its update is an MMA
// accumulation; its bf16 copy is written once per chunk as the B operand of U and O. Every
// bf16 tile sits in shared memory with a 128-byte XOR swizzle so that ldmatrix is
// conflict-free. The decay e^{G_C} is folded into the state at the start of the next chunk.
#include "kernels.h"
#include "ptx.cuh"
#include "../../include/hmd.h"

namespace hmd {
namespace {

__device__ unsigned int g_err;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 256;

// shared-memory map (bytes from a 1024-aligned base). 128-column bf16 tiles are two halves of
// [rows][128 B]; 64-column tiles one half.
constexpr uint32_t OFF_KT = 0;        // Kt  [64][128]
constexpr uint32_t OFF_QT = 16384;    // Qt  [64][128]
constexpr uint32_t OFF_KH = 32768;    // Kh  [64][128]
constexpr uint32_t OFF_V = 49152;     // V   [64][128]
constexpr uint32_t OFF_NW = 65536;    // -W  [64][128]
constexpr uint32_t OFF_U = 81920;     // U   [64][128]
constexpr uint32_t OFF_M = 98304;     // M   [128][128] (bf16 copy of the state)
constexpr uint32_t OFF_T = 131072;    // T   [64][64]
constexpr uint32_t OFF_P = 139264;    // P   [64][64]
constexpr uint32_t OFF_AS = 147456;   // A   fp32 [64][68]
constexpr uint32_t OFF_XS = 164864;   // X   fp32 [64][68]
constexpr uint32_t OFF_YS = 182272;   // Y   fp32 [3][16][20]
constexpr uint32_t OFF_SMALL = 186112;
constexpr uint32_t SMEM_BYTES = OFF_SMALL + 4096 + 1024;
// the raw KDA log-gate tile [64][128] fp32 is staged in the A/X region (free at that point)
constexpr uint32_t OFF_LG = OFF_AS;
constexpr int AS_LD = 68;
constexpr int YS_LD = 20;

// byte offset of element (row, col) of a tile whose halves (64 columns each) hold `rows` rows
__device__ __forceinline__ uint32_t toff(int row, int col, int rows) {
    return (uint32_t)((col >> 6) * rows * 128 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                      ((col & 7) << 1));
}

__device__ __forceinline__ void st_bf16x2(uint8_t *base, uint32_t off, float lo, float hi) {
    *reinterpret_cast<uint32_t *>(base + off) = pack_bf16x2(lo, hi);
}

template <bool KDA>
__global__ void __launch_bounds__(kThreads, 1) prefill_mma_kernel(const DeltaPrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    float *As = reinterpret_cast<float *>(sm + OFF_AS);
    float *Xs = reinterpret_cast<float *>(sm + OFF_XS);
    float *Ys = reinterpret_cast<float *>(sm + OFF_YS);
    float *sbeta = reinterpret_cast<float *>(sm + OFF_SMALL);  // [64]
    float *gam_prev = sbeta + 64;                               // [128]
    float *gam_cur = gam_prev + 128;                            // [128]
    float *etok = gam_cur + 128;                                // [64]
    float *ietok = etok + 64;                                   // [64]
    float *wsum = ietok + 64;                                   // [2]
    float *hsum = wsum + 2;                                     // [2][128] half-chunk gate sums

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int bh = blockIdx.x, b = bh / a.H, h = bh - b * a.H;
    const int T = a.T;
    const int slot = a.slots ? a.slots[b] : b;
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) atomicOr(&g_err, HMD_DEVERR_SLOT);
        return;
    }
    float *Mg = a.state + ((size_t)slot * a.H + h) * kD * kD;
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q);
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(a.k);
    const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(a.v);
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o);

    // the state strip of this warp: rows 16*warp + g (+8), columns 8*nt + 2*t4 (+1)
    const int sr0 = 16 * warp + g, sr1 = sr0 + 8;
    float st[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
        const float2 x0 = *reinterpret_cast<const float2 *>(Mg + (size_t)sr0 * kD + nt * 8 + 2 * t4);
        const float2 x1 = *reinterpret_cast<const float2 *>(Mg + (size_t)sr1 * kD + nt * 8 + 2 * t4);
        st[nt][0] = x0.x; st[nt][1] = x0.y; st[nt][2] = x1.x; st[nt][3] = x1.y;
    }
    if (tid < kD) gam_prev[tid] = 1.f;

    // ldmatrix lane roles
    const int l7 = lane & 7, lb3 = (lane >> 3) & 1, lb4 = lane >> 4;

    for (int t0 = 0; t0 < T; t0 += kC) {
        const int n = min(kC, T - t0);
        // ---- stage the chunk's inputs in shared memory: q (into the Qt slot), k (into the Kh
        //      slot), v, KDA log-gates; beta and per-token GDN gate prefixes ------------------
        {
            const size_t row0 = ((size_t)b * T + t0) * a.H + h;  // token t0's row in [B][T][H]
            // all loads first (independent, 16 bytes each), then all shared-memory stores
            uint4 qv[4], kv[4], vv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int idx = tid + j * kThreads, r = idx >> 4, ch = idx & 15;
                qv[j] = kv[j] = vv[j] = make_uint4(0, 0, 0, 0);
                if (r < n) {
                    const size_t off = (row0 + (size_t)r * a.H) * kD + ch * 8;
                    qv[j] = __ldg(reinterpret_cast<const uint4 *>(qg + off));
                    kv[j] = __ldg(reinterpret_cast<const uint4 *>(kg + off));
                    vv[j] = __ldg(reinterpret_cast<const uint4 *>(vg + off));
                }
            }
            float4 gv[8];
            if constexpr (KDA) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int idx = tid + j * kThreads, r = idx >> 5, c4 = idx & 31;
                    gv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (r < n)
                        gv[j] = __ldg(reinterpret_cast<const float4 *>(a.log_gate + (row0 + (size_t)r * a.H) * kD + c4 * 4));
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int idx = tid + j * kThreads, r = idx >> 4, ch = idx & 15;
                const uint32_t o = toff(r, ch * 8, 64);
                *reinterpret_cast<uint4 *>(sm + OFF_QT + o) = qv[j];
                *reinterpret_cast<uint4 *>(sm + OFF_KH + o) = kv[j];
                *reinterpret_cast<uint4 *>(sm + OFF_V + o) = vv[j];
            }
            if constexpr (KDA) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int idx = tid + j * kThreads, r = idx >> 5, c4 = idx & 31;
                    *reinterpret_cast<float4 *>(sm + OFF_LG + r * 512 + c4 * 16) = gv[j];
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
                    etok[tid] = x;
                }
            }
        }
        __syncthreads();
        // ---- gate pass: Kt, Qt, Kh and e^{G_C}; thread (channel i, token half hf) ---------------
        {
            const int i = tid & (kD - 1), hf = tid >> 7;
            const float *lgs = reinterpret_cast<const float *>(sm + OFF_LG) + i;
            if constexpr (KDA) {
                float part = 0.f;
#pragma unroll 8
                for (int r = 32 * hf; r < 32 * hf + 32; ++r) part += lgs[r * kD];
                hsum[hf * kD + i] = part;
            } else {
                if (tid < kC) {
                    const float gc = etok[tid] + (warp == 1 ? wsum[0] : 0.f);
                    etok[tid] = expf(gc);
                    ietok[tid] = expf(-gc);
                }
            }
            __syncthreads();
            float gsum = KDA ? (hf ? hsum[i] : 0.f) : 0.f;
#pragma unroll 4
            for (int r = 32 * hf; r < 32 * hf + 32; ++r) {
                float e, ie;
                if constexpr (KDA) {
                    gsum += lgs[r * kD];
                    e = expf(gsum);
                    ie = expf(-gsum);
                } else {
                    e = etok[r];
                    ie = ietok[r];
                }
                const uint32_t o = toff(r, i, 64);
                const float kv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_KH + o));
                const float qv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_QT + o));
                *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_KT + o) = __float2bfloat16_rn(kv * e);
                *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_QT + o) = __float2bfloat16_rn(qv * e);
                *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_KH + o) = __float2bfloat16_rn(kv * ie);
            }
            if (hf == 1) gam_cur[i] = KDA ? expf(gsum) : etok[kC - 1];
        }
        __syncthreads();

        // ---- A (warps 0-3) and P (warps 4-7), 16 rows each: [Kt | Qt] Kh^T -------------------
        {
            const int mat = warp >> 2, rt = warp & 3;
            const uint32_t abase = sb + (mat ? OFF_QT : OFF_KT);
            float acc[8][4];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
                uint32_t af[4];
                ldmatrix_x4(abase + toff(16 * rt + l7 + lb3 * 8, kk * 16 + lb4 * 8, 64), af[0], af[1],
                            af[2], af[3]);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(sb + OFF_KH + toff(np * 16 + l7 + lb4 * 8, kk * 16 + lb3 * 8, 64), b0, b1,
                                b2, b3);
                    mma_bf16_16816(acc[2 * np], af, b0, b1);
                    mma_bf16_16816(acc[2 * np + 1], af, b2, b3);
                }
            }
            const int r0 = 16 * rt + g, r1 = r0 + 8;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int s0 = nt * 8 + 2 * t4;
                if (mat == 0) {
                    As[r0 * AS_LD + s0] = (s0 < r0 && r0 < n) ? sbeta[r0] * acc[nt][0] : 0.f;
                    As[r0 * AS_LD + s0 + 1] = (s0 + 1 < r0 && r0 < n) ? sbeta[r0] * acc[nt][1] : 0.f;
                    As[r1 * AS_LD + s0] = (s0 < r1 && r1 < n) ? sbeta[r1] * acc[nt][2] : 0.f;
                    As[r1 * AS_LD + s0 + 1] = (s0 + 1 < r1 && r1 < n) ? sbeta[r1] * acc[nt][3] : 0.f;
                } else {
                    st_bf16x2(sm + OFF_P, toff(r0, s0, 64), (s0 <= r0 && r0 < n) ? acc[nt][0] : 0.f,
                              (s0 + 1 <= r0 && r0 < n) ? acc[nt][1] : 0.f);
                    st_bf16x2(sm + OFF_P, toff(r1, s0, 64), (s0 <= r1 && r1 < n) ? acc[nt][2] : 0.f,
                              (s0 + 1 <= r1 && r1 < n) ? acc[nt][3] : 0.f);
                }
            }
        }
        __syncthreads();

        // ---- X = (I + A)^-1 (16x16 blocks), T = X Diag(beta) ----------------------------------
        if (tid < 64) {
            const int bi = tid >> 4, c0 = tid & 15;
            const float *ab = As + bi * 16 * AS_LD + bi * 16;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int s = 0; s < r; ++s) acc += ab[r * AS_LD + s] * x[s];
                x[r] = r < c0 ? 0.f : (r == c0 ? 1.f : -acc);
                Xs[(bi * 16 + r) * AS_LD + bi * 16 + c0] = x[r];
            }
        }
        __syncthreads();
#pragma unroll 1
        for (int L = 1; L < 4; ++L) {
            const int nb = 4 - L;
            for (int it = tid; it < nb * 64; it += kThreads) {
                const int j = it >> 6, r = (it >> 2) & 15, cg = it & 3, i = j + L;
                const float *arow = As + (i * 16 + r) * AS_LD;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int k = j * 16; k < i * 16; ++k) {
                    const float av = arow[k];
                    const float4 xv = *reinterpret_cast<const float4 *>(Xs + k * AS_LD + j * 16 + cg * 4);
                    acc.x += av * xv.x; acc.y += av * xv.y; acc.z += av * xv.z; acc.w += av * xv.w;
                }
                *reinterpret_cast<float4 *>(Ys + (j * 16 + r) * YS_LD + cg * 4) = acc;
            }
            __syncthreads();
            for (int it = tid; it < nb * 64; it += kThreads) {
                const int j = it >> 6, r = (it >> 2) & 15, cg = it & 3, i = j + L;
                const float *xrow = Xs + (i * 16 + r) * AS_LD + i * 16;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int s = 0; s <= r; ++s) {
                    const float xv = xrow[s];
                    const float4 yv = *reinterpret_cast<const float4 *>(Ys + (j * 16 + s) * YS_LD + cg * 4);
                    acc.x += xv * yv.x; acc.y += xv * yv.y; acc.z += xv * yv.z; acc.w += xv * yv.w;
                }
                *reinterpret_cast<float4 *>(Xs + (i * 16 + r) * AS_LD + j * 16 + cg * 4) =
                    make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
            }
            __syncthreads();
        }
        for (int idx = tid; idx < 64 * 32; idx += kThreads) {
            const int r = idx >> 5, s0 = (idx & 31) * 2;
            const float v0 = s0 <= r ? Xs[r * AS_LD + s0] * sbeta[s0] : 0.f;
            const float v1 = s0 + 1 <= r ? Xs[r * AS_LD + s0 + 1] * sbeta[s0 + 1] : 0.f;
            st_bf16x2(sm + OFF_T, toff(r, s0, 64), v0, v1);
        }
        __syncthreads();

        // ---- Ut = T V (warps 0-3, kept in registers) and W = T Kt (warps 4-7, stored as -W) ----
        const int mat = warp >> 2, rt = warp & 3;
        float acc[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
        {
            const uint32_t bbase = sb + (mat ? OFF_KT : OFF_V);
#pragma unroll
            for (int kk = 0; kk < kC / 16; ++kk) {
                uint32_t af[4];
                ldmatrix_x4(sb + OFF_T + toff(16 * rt + l7 + lb3 * 8, kk * 16 + lb4 * 8, 64), af[0], af[1],
                            af[2], af[3]);
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(bbase + toff(kk * 16 + l7 + lb3 * 8, np * 16 + lb4 * 8, 64), b0, b1,
                                      b2, b3);
                    mma_bf16_16816(acc[2 * np], af, b0, b1);
                    mma_bf16_16816(acc[2 * np + 1], af, b2, b3);
                }
            }
        }
        if (mat == 1) {
            const int r0 = 16 * rt + g, r1 = r0 + 8;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                const int c = nt * 8 + 2 * t4;
                st_bf16x2(sm + OFF_NW, toff(r0, c, 64), -acc[nt][0], -acc[nt][1]);
                st_bf16x2(sm + OFF_NW, toff(r1, c, 64), -acc[nt][2], -acc[nt][3]);
                acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
            }
        }
        // ---- state pass: M = Diag(e^{G_prev}) Mraw (registers) and its bf16 copy ------------
        {
            const float gp0 = gam_prev[sr0], gp1 = gam_prev[sr1];
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                st[nt][0] *= gp0; st[nt][1] *= gp0; st[nt][2] *= gp1; st[nt][3] *= gp1;
                const int c = nt * 8 + 2 * t4;
                st_bf16x2(sm + OFF_M, toff(sr0, c, 128), st[nt][0], st[nt][1]);
                st_bf16x2(sm + OFF_M, toff(sr1, c, 128), st[nt][2], st[nt][3]);
            }
        }
        __syncthreads();

        // ---- U = Ut + (-W) M (warps 0-3)  and  O = Qt M (warps 4-7) --------------------------
        {
            const uint32_t abase = sb + (mat ? OFF_QT : OFF_NW);
#pragma unroll 2
            for (int kk = 0; kk < kD / 16; ++kk) {
                uint32_t af[4];
                ldmatrix_x4(abase + toff(16 * rt + l7 + lb3 * 8, kk * 16 + lb4 * 8, 64), af[0], af[1], af[2],
                            af[3]);
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(sb + OFF_M + toff(kk * 16 + l7 + lb3 * 8, np * 16 + lb4 * 8, 128), b0,
                                      b1, b2, b3);
                    mma_bf16_16816(acc[2 * np], af, b0, b1);
                    mma_bf16_16816(acc[2 * np + 1], af, b2, b3);
                }
            }
        }
        if (mat == 0) {
            const int r0 = 16 * rt + g, r1 = r0 + 8;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                const int c = nt * 8 + 2 * t4;
                st_bf16x2(sm + OFF_U, toff(r0, c, 64), acc[nt][0], acc[nt][1]);
                st_bf16x2(sm + OFF_U, toff(r1, c, 64), acc[nt][2], acc[nt][3]);
            }
        }
        __syncthreads();

        // ---- O += P U, then store (warps 4-7) ------------------------------------------------
        if (mat == 1) {
#pragma unroll
            for (int kk = 0; kk < kC / 16; ++kk) {
                uint32_t af[4];
                ldmatrix_x4(sb + OFF_P + toff(16 * rt + l7 + lb3 * 8, kk * 16 + lb4 * 8, 64), af[0], af[1],
                            af[2], af[3]);
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(sb + OFF_U + toff(kk * 16 + l7 + lb3 * 8, np * 16 + lb4 * 8, 64), b0, b1,
                                      b2, b3);
                    mma_bf16_16816(acc[2 * np], af, b0, b1);
                    mma_bf16_16816(acc[2 * np + 1], af, b2, b3);
                }
            }
            const int r0 = 16 * rt + g, r1 = r0 + 8;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                const int c = nt * 8 + 2 * t4;
                if (r0 < n)
                    *reinterpret_cast<uint32_t *>(og + (((size_t)b * T + t0 + r0) * a.H + h) * kD + c) =
                        pack_bf16x2(a.scale * acc[nt][0], a.scale * acc[nt][1]);
                if (r1 < n)
                    *reinterpret_cast<uint32_t *>(og + (((size_t)b * T + t0 + r1) * a.H + h) * kD + c) =
                        pack_bf16x2(a.scale * acc[nt][2], a.scale * acc[nt][3]);
            }
        }
        // ---- Mraw = M + Kh^T U (every warp, its 16-row strip) ---------------------------------
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk) {
            uint32_t af[4];
            ldmatrix_x4_trans(sb + OFF_KH + toff(kk * 16 + l7 + lb4 * 8, 16 * warp + lb3 * 8, 64), af[0],
                              af[1], af[2], af[3]);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(sb + OFF_U + toff(kk * 16 + l7 + lb3 * 8, np * 16 + lb4 * 8, 64), b0, b1, b2,
                                  b3);
                mma_bf16_16816(st[2 * np], af, b0, b1);
                mma_bf16_16816(st[2 * np + 1], af, b2, b3);
            }
        }
        if (tid < kD) gam_prev[tid] = gam_cur[tid];
        __syncthreads();
    }
    // final state Diag(e^{G_C}) Mraw
    {
        const float gp0 = gam_prev[sr0], gp1 = gam_prev[sr1];
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            *reinterpret_cast<float2 *>(Mg + (size_t)sr0 * kD + nt * 8 + 2 * t4) =
                make_float2(st[nt][0] * gp0, st[nt][1] * gp0);
            *reinterpret_cast<float2 *>(Mg + (size_t)sr1 * kD + nt * 8 + 2 * t4) =
                make_float2(st[nt][2] * gp1, st[nt][3] * gp1);
        }
    }
}

}  // namespace

bool delta_prefill_mma_supported(int dk, int dv, bool bf16, int chunk) {
    return bf16 && dk == kD && dv == kD && chunk == kC;
}

cudaError_t launch_delta_prefill_mma(const DeltaPrefillArgs &a, cudaStream_t s) {
    static cudaError_t attr = [] {
        cudaError_t e = cudaFuncSetAttribute(prefill_mma_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(prefill_mma_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        return e;
    }();
    if (attr != cudaSuccess) return attr;
    const unsigned grid = (unsigned)(a.B * a.H);
    if (a.kind == HMD_KDA)
        prefill_mma_kernel<true><<<grid, kThreads, SMEM_BYTES, s>>>(a);
    else
        prefill_mma_kernel<false><<<grid, kThreads, SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

uint32_t delta_prefill_mma_read_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_err, sizeof v) != cudaSuccess) return 0;
    if (clear && v) {
        const unsigned int z = 0;
        cudaMemcpyToSymbol(g_err, &z, sizeof z);
    }
    return v;
}

}  // namespace hmd

// FA / SWA prefill on the 5th-generation tensor cores (tcgen05, TMEM), d = 128.
//
// Same operation, layouts and cache write as attn_prefill.cu (FA and SWA from the gist.science
// technical summary of "Super Apriel: One Checkpoint, Many Speeds", sections 1 and 2a): token t
// attends keys [lo_t, t], lo_t = 0 (FA) or max(0, t + 1 - w) (SWA).
//
// One CTA of 8 warps per (sequence, kv-head, block of 128/G tokens). Query row r (head
// g*G + r / QT, token t_first + r % QT) is TMEM lane r of every accumulator; threads r and
// r + 128 (warps w and w + 4 read the same TMEM lanes) split its columns: each takes half of the
// row's scores and half of its output, and they exchange one partial maximum per tile. Per
// 64-key tile i:
//   S_i = Q K_i^T   tcgen05.mma M=128 N=64 K=128 (Q and K K-major, 128-byte swizzle) into one
//                   of two TMEM buffers; issued one tile ahead so it overlaps the softmax
//   softmax         tcgen05.ld of the row, online max / sum in the log2 domain, P_i in bf16 to
//                   shared memory in the swizzled K-major layout (two buffers)
//   PV_i = P_i V_i  tcgen05.mma M=128 N=128 K=64 (V MN-major) into TMEM; the next tile reads it
//                   back and folds it into the fp32 O accumulator held in registers.
// The accumulators are only ever read from TMEM (tcgen05.ld), never written by the threads. One
// thread issues the TMA copies (3-stage K/V ring, 3-D boxes from the prompt) and the MMAs;
// every mbarrier wait is bounded.
#include <cuda.h>
#include <float.h>

#include <mutex>

#include "kernels.h"
#include "ptx.cuh"
#include "../../include/hmd.h"

namespace hmd {
namespace {

__device__ unsigned int g_err;

constexpr int kD = 128;
constexpr int kPT = 64;        // keys per tile = tokens per page
constexpr int kStages = 3;     // K/V tiles in flight
constexpr int kThreads = 256;  // threads r and r + 128 share query row r = TMEM lane r
constexpr int kRows = 128;
constexpr uint32_t kTmemCols = 256;  // S buffers at 0 and 64, PV at 128

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;                  // Q [128 rows][128 dims]: 2 halves of 16 KiB
constexpr uint32_t OFF_KV = 32768;             // stage s: K at +0, V at +16384 (2 halves each)
constexpr uint32_t STAGE = 32768;
constexpr uint32_t OFF_P = OFF_KV + kStages * STAGE;  // P [128 rows][64 keys] x 2 buffers
constexpr uint32_t P_BYTES = 16384;
constexpr uint32_t OFF_RED = OFF_P + 2 * P_BYTES;     // partial row maxima [2][128] fp32
constexpr uint32_t OFF_BAR = OFF_RED + 1024;          // full[3], s_done[2], pv_done, tmem slot
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;

constexpr uint32_t ID_S = idesc_bf16(128, 64, 0, 0);    // A = Q (K-major), B = K (K-major)
constexpr uint32_t ID_PV = idesc_bf16(128, 128, 0, 1);  // A = P (K-major), B = V (MN-major)

struct TcParams {
    const __nv_bfloat16 *q, *k, *v;
    __nv_bfloat16 *k_pool, *v_pool, *o;
    const int32_t *page_table;
    int B, T, Hq, Hkv, G, QT, n_qb;
    int window, swa, ring_pages, max_pages, n_pages;
    float scale_log2;
};

// byte offset of (row, col..col+7) in [rows][128 B] blocks of 64 columns, 128-byte swizzle
__device__ __forceinline__ uint32_t swz(int row, int col, int rows) {
    return (uint32_t)((col >> 6) * rows * 128 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4));
}

__device__ __forceinline__ int key_lo(const TcParams &p, int t) {
    return (p.swa && t + 1 > p.window) ? t + 1 - p.window : 0;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                       const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    const uint32_t bar_full = smem_u32(&bars[0]);    // + 8 * stage
    const uint32_t bar_s = smem_u32(&bars[3]);       // + 8 * (tile & 1)
    const uint32_t bar_pv = smem_u32(&bars[5]);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 48);
    const int tid = threadIdx.x, warp = tid >> 5;

    const int bg = blockIdx.x % (p.B * p.Hkv);
    const int qb = p.n_qb - 1 - (int)(blockIdx.x / (p.B * p.Hkv));  // longest blocks first
    const int b = bg / p.Hkv, g = bg - b * p.Hkv;
    const int t_first = qb * p.QT;
    const int t_last = min(p.T, t_first + p.QT) - 1;

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(smem_u32(&bars[i]), 1);
        fence_barrier_init();
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    griddep_launch_dependents();
    griddep_wait();  // the prompt and the cache may come from the previous kernel
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);

    const int kb_lo = key_lo(p, t_first) / kPT, kb_hi = t_last / kPT;
    const int n_tiles = kb_hi - kb_lo + 1;
    auto issue_tile = [&](int i) {  // thread 0
        const int s = i % kStages;
        const uint32_t bar = bar_full + 8 * s;
        mbar_arrive_expect_tx(bar, STAGE);  // K and V tiles: 4 boxes of 8 KiB
        const uint32_t kb = sb + OFF_KV + s * STAGE, vb = kb + 16384;
        const int z = b * p.T + (kb_lo + i) * kPT;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(kb + hf * 8192, &tmk, bar, hf * 64, g, z);
            tma_load_3d(vb + hf * 8192, &tmv, bar, hf * 64, g, z);
        }
    };
    int tiles_issued = 0, s_issued = 0, pv_issued = 0;  // thread 0's bookkeeping
    if (tid == 0)
        for (; tiles_issued < 2 && tiles_issued < n_tiles; ++tiles_issued) issue_tile(tiles_issued);

    // ---- row r = tid % 128 (its token, head and window); column half ch = tid / 128 ---------
    const int row = tid & (kRows - 1), ch = tid >> 7;
    const int t_row = t_first + row % p.QT;
    const bool row_ok = t_row <= t_last;
    const int lo_row = key_lo(p, t_row);
    const int h_row = g * p.G + row / p.QT;
    float *red = reinterpret_cast<float *>(sm + OFF_RED);  // [2][128]

    // Q row -> shared memory (swizzled K-major A operand), half a row per thread; zero past the
    // prompt
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(
            p.q + (((size_t)b * p.T + (row_ok ? t_row : 0)) * p.Hq + h_row) * kD);
#pragma unroll
        for (int c = ch * 8; c < ch * 8 + 8; ++c) {
            const uint4 v = row_ok ? src[c] : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sm + OFF_Q + swz(row, c * 8, kRows)) = v;
        }
    }
    // ---- fused cache write: this block's tokens of kv-head g (as attn_prefill.cu) -------------
    {
        const int ring = p.ring_pages * kPT;
        const int n_tok = t_last - t_first + 1;
        constexpr int CH = kD / 8;
        for (int idx = tid; idx < n_tok * 2 * CH; idx += kThreads) {
            const int tt = idx / (2 * CH), rem = idx - tt * 2 * CH;
            const bool is_v = rem >= CH;
            const int ch = is_v ? rem - CH : rem;
            const int t = t_first + tt;
            if (p.swa && t < p.T - ring) continue;
            const int li = p.swa ? t % ring : t;
            const int lp = li / kPT;
            const int pg = lp < p.max_pages ? p.page_table[(size_t)b * p.max_pages + lp] : -1;
            if (pg < 0 || pg >= p.n_pages) {
                atomicOr(&g_err, HMD_DEVERR_PAGE);
                continue;
            }
            const size_t srco = (((size_t)b * p.T + t) * p.Hkv + g) * kD + ch * 8;
            const size_t dsto = (((size_t)pg * p.Hkv + g) * kPT + (li % kPT)) * kD + ch * 8;
            *reinterpret_cast<uint4 *>((is_v ? p.v_pool : p.k_pool) + dsto) =
                *reinterpret_cast<const uint4 *>((is_v ? p.v : p.k) + srco);
        }
    }
    fence_proxy_async_smem();  // Q is read by the tensor cores
    __syncthreads();

    auto issue_s = [&](int i) {  // thread 0: S_i = Q K_i^T -> TMEM buffer i & 1
        const uint32_t kbase = sb + OFF_KV + (i % kStages) * STAGE;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(sb + OFF_Q + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(kbase + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
            umma_bf16(tmem + (i & 1) * 64, ad, bd, ID_S, kk > 0);
        }
        umma_commit(bar_s + 8 * (i & 1));
    };
    auto issue_pv = [&](int i) {  // thread 0: PV_i = P_i V_i -> TMEM columns 128..255
        const uint32_t pbase = sb + OFF_P + (i & 1) * P_BYTES;
        const uint32_t vbase = sb + OFF_KV + (i % kStages) * STAGE + 16384;
#pragma unroll
        for (int kk = 0; kk < kPT / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(pbase + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(vbase + kk * 2048, 8192, 1024);
            umma_bf16(tmem + 128, ad, bd, ID_PV, kk > 0);
        }
        umma_commit(bar_pv);
    };

    bool fail = false;
    if (tid == 0) {
        if (mbar_wait_bounded(bar_full, 0)) {
            tc_fence_after();
            issue_s(0);
            s_issued = 1;
        } else {
            fail = true;
        }
    }

    float o[kD / 2];  // this thread's half of the row's output
#pragma unroll
    for (int j = 0; j < kD / 2; ++j) o[j] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;  // l_run: this thread's half of the row sum

    int i = 0;
    for (; i < n_tiles; ++i) {
        // ---- this thread's 32 scores of S_i -> registers ------------------------------------
        float s[kPT / 2];
        if (!fail) {
            if (!mbar_wait_bounded(bar_s + 8 * (i & 1), (i >> 1) & 1)) fail = true;
        }
        if (!fail) {
            tc_fence_after();
            uint32_t r[32];
            tmem_ld32(lane_base + (i & 1) * 64 + ch * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) s[j] = __uint_as_float(r[j]);
        }
        // ---- thread 0: S_{i+1} into the other buffer (read by every thread last iteration) ---
        if (tid == 0 && !fail && i + 1 < n_tiles) {
            const int n1 = i + 1;
            if (mbar_wait_bounded(bar_full + 8 * (n1 % kStages), (n1 / kStages) & 1)) {
                tc_fence_after();
                issue_s(n1);
                ++s_issued;
            } else {
                fail = true;
            }
        }
        // ---- mask, scale, partial maximum of this half row -----------------------------------
        const int j0 = (kb_lo + i) * kPT + ch * 32;
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < kPT / 2; ++j) {
            const int key = j0 + j;
            const bool valid = row_ok && key >= lo_row && key <= t_row;
            s[j] = valid ? s[j] * p.scale_log2 : -INFINITY;
            mx = fmaxf(mx, s[j]);
        }
        red[ch * kRows + row] = mx;
        __syncthreads();
        // ---- softmax with the row's maximum; P_i half row -> shared memory -------------------
        const float m_new = fmaxf(m_run, fmaxf(red[row], red[kRows + row]));
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        const float corr = exp2f(m_run - mu);
        m_run = m_new;
        {
            float ls = 0.f;
            uint8_t *prow = sm + OFF_P + (i & 1) * P_BYTES;
#pragma unroll
            for (int c = 0; c < kPT / 16; ++c) {
                float e[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    e[u] = exp2f(s[c * 8 + u] - mu);
                    ls += e[u];
                }
                *reinterpret_cast<uint4 *>(prow + swz(row, ch * 32 + c * 8, kRows)) =
                    make_uint4(pack_bf16x2(e[0], e[1]), pack_bf16x2(e[2], e[3]),
                               pack_bf16x2(e[4], e[5]), pack_bf16x2(e[6], e[7]));
            }
            l_run = l_run * corr + ls;
        }
        // ---- PV_{i-1} (scale of tile i-1) joins O; then O takes this tile's scale ------------
        if (i > 0 && !fail) {
            if (!mbar_wait_bounded(bar_pv, (i - 1) & 1)) fail = true;
        }
        if (i > 0 && !fail) {
            tc_fence_after();
#pragma unroll
            for (int c4 = 0; c4 < kD / 64; ++c4) {
                uint32_t r[32];
                tmem_ld32(lane_base + 128 + ch * 64 + c4 * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) o[c4 * 32 + j] = (o[c4 * 32 + j] + __uint_as_float(r[j])) * corr;
            }
        }
        // ---- thread 0: tile i+2 into the stage tile i-1 used (its S and PV are done) ----------
        if (tid == 0 && !fail && tiles_issued < n_tiles && tiles_issued <= i + 2) {
            issue_tile(tiles_issued);
            ++tiles_issued;
        }
        // ---- every thread has written P_i and read S_i, PV_{i-1} and the maxima --------------
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(fail)) break;
        if (tid == 0) {
            tc_fence_after();
            issue_pv(i);
            ++pv_issued;
        }
    }
    const bool aborted = i < n_tiles;
    if (!aborted) {
        // the last PV joins O; the two halves' sums make the row's; normalise and store
        bool ok = mbar_wait_bounded(bar_pv, (n_tiles - 1) & 1);
        red[ch * kRows + row] = l_run;
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
        } else {
            tc_fence_after();
#pragma unroll
            for (int c4 = 0; c4 < kD / 64; ++c4) {
                uint32_t r[32];
                tmem_ld32(lane_base + 128 + ch * 64 + c4 * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) o[c4 * 32 + j] += __uint_as_float(r[j]);
            }
            if (row_ok) {
                const float l = red[row] + red[kRows + row];
                const float inv = l > 0.f ? 1.f / l : 0.f;
                uint4 *dst = reinterpret_cast<uint4 *>(
                    p.o + (((size_t)b * p.T + t_row) * p.Hq + h_row) * kD + ch * 64);
#pragma unroll
                for (int c = 0; c < kD / 16; ++c)
                    dst[c] = make_uint4(pack_bf16x2(o[c * 8] * inv, o[c * 8 + 1] * inv),
                                        pack_bf16x2(o[c * 8 + 2] * inv, o[c * 8 + 3] * inv),
                                        pack_bf16x2(o[c * 8 + 4] * inv, o[c * 8 + 5] * inv),
                                        pack_bf16x2(o[c * 8 + 6] * inv, o[c * 8 + 7] * inv));
            }
        }
    } else if (tid == 0) {
        // a wait gave up: let what this CTA started finish (bounded) before freeing TMEM
        atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
        if (s_issued > 0)
            (void)mbar_wait_bounded(bar_s + 8 * ((s_issued - 1) & 1), ((s_issued - 1) >> 1) & 1);
        if (pv_issued > 0) (void)mbar_wait_bounded(bar_pv, (pv_issued - 1) & 1);
        for (int u = max(0, tiles_issued - kStages); u < tiles_issued; ++u)
            (void)mbar_wait_bounded(bar_full + 8 * (u % kStages), (u / kStages) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool attn_prefill_tc_supported(int d, int page_tokens, int group) {
    const bool g_ok = group == 1 || group == 2 || group == 4 || group == 8 || group == 16;
    return d == kD && page_tokens == kPT && g_ok;
}

cudaError_t launch_attn_prefill_tc(const AttnPrefillArgs &a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(attn_prefill_tc_kernel,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap tmk, tmv;
    const long long n_tok = (long long)a.B * a.T;
    if (!make_tmap_tokens_sw128(&tmk, const_cast<void *>(a.k), n_tok, a.Hkv, kD) ||
        !make_tmap_tokens_sw128(&tmv, const_cast<void *>(a.v), n_tok, a.Hkv, kD))
        return cudaErrorInvalidValue;
    TcParams p;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.k = static_cast<const __nv_bfloat16 *>(a.k);
    p.v = static_cast<const __nv_bfloat16 *>(a.v);
    p.k_pool = static_cast<__nv_bfloat16 *>(a.k_pool);
    p.v_pool = static_cast<__nv_bfloat16 *>(a.v_pool);
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.page_table = a.page_table;
    p.B = a.B; p.T = a.T; p.Hq = a.Hq; p.Hkv = a.Hkv;
    p.G = a.Hq / a.Hkv;
    p.QT = kRows / p.G;
    p.n_qb = (a.T + p.QT - 1) / p.QT;
    p.window = a.window; p.swa = a.swa ? 1 : 0;
    p.ring_pages = a.swa ? (a.window + kPT - 1) / kPT : 0;
    p.max_pages = a.max_pages; p.n_pages = a.n_pages;
    p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
    const long long grid = (long long)p.n_qb * a.B * a.Hkv;
    return launch_pdl(attn_prefill_tc_kernel, dim3((unsigned)grid), dim3(kThreads), SMEM_BYTES, s,
                      tmk, tmv, p);
}

uint32_t attn_prefill_tc_read_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_err, sizeof v) != cudaSuccess) return 0;
    if (clear && v) {
        const unsigned int z = 0;
        cudaMemcpyToSymbol(g_err, &z, sizeof z);
    }
    return v;
}

}  // namespace hmd

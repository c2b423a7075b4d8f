// FA / SWA prefill: causal (or windowed) GQA attention over a prompt of T tokens per sequence,
// from an empty cache, with the prompt's K and V written into the paged cache.
//
// FA is causal attention whose KV cache grows with the context, SWA attends to the last w keys
// (gist.science technical summary of "Super Apriel: One Checkpoint, Many Speeds", sections 1
// and 2a). Token t of sequence b sits at logical position t and attends keys j in [lo_t, t],
// lo_t = 0 (FA) or max(0, t + 1 - w) (SWA): the decode step with L = t + 1, for every t at once.
// Query head h reads kv-head h / (Hq / Hkv).
//
// One CTA per (sequence, kv-head, block of query tokens): its 128 query rows are the GQA
// group's G heads x 128/G tokens, so every K/V tile it loads serves all heads of the group. The
// tiles (64 keys) come from the prompt's own K and V by 3-D TMA boxes with the 128-byte swizzle
// through a 2-stage ring (two CTAs per SM); each of the 4 warps takes 32 query rows as two m16
// tiles that share every K and V fragment it loads (half the shared-memory reads per flop of
// one tile per warp): S = Q K^T and O += P V on mma.sync m16n8k16 (bf16, fp32 accumulate) with
// an online softmax in the log2 domain; Q sits in shared memory. Only
// tiles on the causal diagonal or the window's lower edge are masked; a warp skips a tile none
// of its rows can see. Query blocks are scheduled longest first.
// The cache write is fused: each CTA copies its own tokens' K and V of its kv-head to their
// slots (FA: page_table[b][t / 64], t % 64; SWA: ring index t mod (R*64), R = ceil(w / 64),
// only the positions the ring keeps, t >= T - R*64), so every slot is written once.
#include <cuda.h>
#include <float.h>

#include <climits>
#include <mutex>

#include "kernels.h"
#include "ptx.cuh"
#include "../../include/hmd.h"

namespace hmd {
namespace {

__device__ unsigned int g_err;

constexpr int kPT = 64;        // tokens per page = keys per tile
constexpr int kStages = 2;     // K/V tiles in flight per CTA (two CTAs per SM)
constexpr int kThreads = 128;  // 4 warps x 32 query rows
constexpr int kRows = 128;     // query rows per CTA: G heads x (128 / G) tokens
constexpr int kMT = 2;         // m16 tiles per warp

struct PrefillParams {
    const __nv_bfloat16 *q, *k, *v;
    __nv_bfloat16 *k_pool, *v_pool, *o;
    const int32_t *page_table;
    int B, T, Hq, Hkv, G, QT, n_qb;
    int window, swa, ring_pages, max_pages, n_pages;
    float scale_log2;  // log2(e) / sqrt(d)
};

// Byte offset of the 16-byte chunk holding (row, dim..dim+7) in a tile of `rows` rows stored as
// D/64 halves of [rows][128 B] with the 128-byte swizzle (chunk index ^= row % 8).
__device__ __forceinline__ uint32_t tile_off(int row, int dim, int rows) {
    return (uint32_t)((dim >> 6) * (rows * 128) + row * 128 + ((((dim & 63) >> 3) ^ (row & 7)) << 4));
}

template <int D>
constexpr int q_bytes() {
    return kRows * D * 2;
}
template <int D>
constexpr int smem_bytes() {
    return kStages * 2 * kPT * D * 2 + q_bytes<D>() + 1024;
}

// first key of token t's window
__device__ __forceinline__ int key_lo(const PrefillParams &p, int t) {
    return (p.swa && t + 1 > p.window) ? t + 1 - p.window : 0;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
attn_prefill_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const PrefillParams p) {
    constexpr int TB = kPT * D * 2;  // bytes of one tile of K or V
    constexpr int NK = D / 16;       // k-steps of Q K^T
    constexpr int NN = D / 8;        // n-tiles of P V
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kStages];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const uint32_t smem_base = smem_u32(smem);
    const uint32_t qs = smem_base + kStages * 2 * TB;  // Q tile [128 rows][D]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // the longest query blocks (the last ones) first
    const int bg = blockIdx.x % (p.B * p.Hkv);
    const int qb = p.n_qb - 1 - (int)(blockIdx.x / (p.B * p.Hkv));
    const int b = bg / p.Hkv, g = bg - b * p.Hkv;
    const int t_first = qb * p.QT;
    const int t_last = min(p.T, t_first + p.QT) - 1;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&full_bar[s]), 1);
        fence_barrier_init();
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    griddep_launch_dependents();
    griddep_wait();  // the prompt and the cache may come from the previous kernel
    __syncthreads();

    const int kb_lo = key_lo(p, t_first) / kPT, kb_hi = t_last / kPT;
    const int n_tiles = kb_hi - kb_lo + 1;
    auto issue = [&](int i) {  // thread 0: tile i -> stage i % kStages
        const int s = i % kStages;
        const uint32_t bar = smem_u32(&full_bar[s]);
        mbar_arrive_expect_tx(bar, 2 * TB);
        const uint32_t kb = smem_base + s * 2 * TB, vb = kb + TB;
        const int z = b * p.T + (kb_lo + i) * kPT;
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
            tma_load_3d(kb + hf * kPT * 128, &tmk, bar, hf * 64, g, z);
            tma_load_3d(vb + hf * kPT * 128, &tmv, bar, hf * 64, g, z);
        }
    };
    if (tid == 0)
        for (int i = 0; i < kStages && i < n_tiles; ++i) issue(i);

    // ---- Q tile: row r is head g*G + r / QT, token t_first + r % QT (zero past the prompt) ---
    {
        constexpr int CH = D / 8;  // 16-byte chunks per row
        for (int idx = tid; idx < kRows * CH; idx += kThreads) {
            const int r = idx / CH, ch = idx - r * CH;
            const int t = t_first + r % p.QT;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (t <= t_last)
                val = *reinterpret_cast<const uint4 *>(
                    p.q + (((size_t)b * p.T + t) * p.Hq + g * p.G + r / p.QT) * D + ch * 8);
            *reinterpret_cast<uint4 *>(smem + kStages * 2 * TB + tile_off(r, ch * 8, kRows)) = val;
        }
    }

    // ---- fused cache write: this block's tokens of kv-head g --------------------------------
    {
        const int ring = p.ring_pages * kPT;
        const int n_tok = t_last - t_first + 1;
        constexpr int CH = D / 8;
        for (int idx = tid; idx < n_tok * 2 * CH; idx += kThreads) {
            const int tt = idx / (2 * CH), rem = idx - tt * 2 * CH;
            const bool is_v = rem >= CH;
            const int ch = is_v ? rem - CH : rem;
            const int t = t_first + tt;
            if (p.swa && t < p.T - ring) continue;  // overwritten later in the ring
            const int li = p.swa ? t % ring : t;
            const int lp = li / kPT;
            const int pg = lp < p.max_pages ? p.page_table[(size_t)b * p.max_pages + lp] : -1;
            if (pg < 0 || pg >= p.n_pages) {
                atomicOr(&g_err, HMD_DEVERR_PAGE);
                continue;
            }
            const size_t src = (((size_t)b * p.T + t) * p.Hkv + g) * D + ch * 8;
            const size_t dst = (((size_t)pg * p.Hkv + g) * kPT + (li % kPT)) * D + ch * 8;
            const uint4 val = *reinterpret_cast<const uint4 *>((is_v ? p.v : p.k) + src);
            *reinterpret_cast<uint4 *>((is_v ? p.v_pool : p.k_pool) + dst) = val;
        }
    }
    __syncthreads();  // Q tile complete

    // ---- this warp's 32 rows: m-tile mt holds rows 32 warp + 16 mt + (lane / 4) (+ 8) --------
    const int cq = (lane & 3) * 2, mi = lane >> 3, l7 = lane & 7;
    int tq[kMT][2];  // token of each of this thread's 4 rows (rows past the prompt see nothing)
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
            tq[mt][h2] = t_first + (32 * warp + 16 * mt + (lane >> 2) + 8 * h2) % p.QT;
    int my_lo = INT_MAX, my_hi = -1;
    bool my_ok = true;
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            if (tq[mt][h2] <= t_last) {
                my_lo = min(my_lo, tq[mt][h2]);
                my_hi = max(my_hi, tq[mt][h2]);
            } else {
                my_ok = false;
            }
        }
    const int t_lo_w = __reduce_min_sync(0xffffffffu, my_lo);
    const int t_hi_w = __reduce_max_sync(0xffffffffu, my_hi);
    const bool all_ok = __all_sync(0xffffffffu, my_ok);
    const int lo_w = t_hi_w >= 0 ? key_lo(p, t_lo_w) : 0;
    const int lo_w_hi = t_hi_w >= 0 ? key_lo(p, t_hi_w) : 0;

    float m_run[kMT][2], l_run[kMT][2];
    float oacc[kMT][NN][4];
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) {
        m_run[mt][0] = m_run[mt][1] = -INFINITY;
        l_run[mt][0] = l_run[mt][1] = 0.f;
#pragma unroll
        for (int n = 0; n < NN; ++n) oacc[mt][n][0] = oacc[mt][n][1] = oacc[mt][n][2] = oacc[mt][n][3] = 0.f;
    }

    for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kStages;
        const bool ok = mbar_wait_bounded(smem_u32(&full_bar[s]), (i / kStages) & 1);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
                // let the copies this CTA issued finish (bounded) before leaving
                for (int u = i; u < n_tiles && u < i + kStages; ++u)
                    (void)mbar_wait_bounded(smem_u32(&full_bar[u % kStages]), (u / kStages) & 1);
            }
            return;  // o is left unwritten; the error word reports the call as failed
        }
        const int j0 = (kb_lo + i) * kPT;
        const bool needed = t_hi_w >= 0 && j0 <= t_hi_w && j0 + kPT - 1 >= lo_w;
        if (needed) {
            const bool masked = !all_ok || j0 + kPT - 1 > t_lo_w || j0 < lo_w_hi;
            const uint32_t kbu = smem_base + s * 2 * TB, vbu = kbu + TB;
            float sc[kMT][8][4];
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
                for (int n = 0; n < 8; ++n) sc[mt][n][0] = sc[mt][n][1] = sc[mt][n][2] = sc[mt][n][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < NK; ++kk) {
                uint32_t qa[kMT][4];
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt)
                    ldmatrix_x4(qs + tile_off(32 * warp + 16 * mt + l7 + ((mi & 1) << 3), kk * 16 + ((mi >> 1) << 3), kRows),
                                qa[mt][0], qa[mt][1], qa[mt][2], qa[mt][3]);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b00, b01, b10, b11;
                    ldmatrix_x4(kbu + tile_off(np * 16 + ((mi >> 1) << 3) + l7, kk * 16 + ((mi & 1) << 3), kPT),
                                b00, b01, b10, b11);
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
                        mma_bf16_16816(sc[mt][2 * np], qa[mt], b00, b01);
                        mma_bf16_16816(sc[mt][2 * np + 1], qa[mt], b10, b11);
                    }
                }
            }
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
                float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int n = 0; n < 8; ++n) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        bool valid = true;
                        if (masked) {
                            const int key = j0 + n * 8 + cq + (e & 1);
                            const int t = tq[mt][e >> 1];
                            valid = t <= t_last && key <= t && key >= key_lo(p, t);
                        }
                        sc[mt][n][e] = valid ? sc[mt][n][e] * p.scale_log2 : -INFINITY;
                        mx[e >> 1] = fmaxf(mx[e >> 1], sc[mt][n][e]);
                    }
                }
                float corr[2], mu[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
                    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
                    const float mnew = fmaxf(m_run[mt][r], mx[r]);
                    mu[r] = (mnew == -INFINITY) ? 0.f : mnew;
                    corr[r] = exp2f(m_run[mt][r] - mu[r]);
                    m_run[mt][r] = mnew;
                }
                float ls[2] = {0.f, 0.f};
#pragma unroll
                for (int n = 0; n < 8; ++n) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        sc[mt][n][e] = exp2f(sc[mt][n][e] - mu[e >> 1]);
                        ls[e >> 1] += sc[mt][n][e];
                    }
                }
                l_run[mt][0] = l_run[mt][0] * corr[0] + ls[0];
                l_run[mt][1] = l_run[mt][1] * corr[1] + ls[1];
#pragma unroll
                for (int n = 0; n < NN; ++n) {
                    oacc[mt][n][0] *= corr[0]; oacc[mt][n][1] *= corr[0];
                    oacc[mt][n][2] *= corr[1]; oacc[mt][n][3] *= corr[1];
                }
            }
#pragma unroll
            for (int kk2 = 0; kk2 < kPT / 16; ++kk2) {
                uint32_t pa[kMT][4];
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                    pa[mt][0] = pack_bf16x2(sc[mt][2 * kk2][0], sc[mt][2 * kk2][1]);
                    pa[mt][1] = pack_bf16x2(sc[mt][2 * kk2][2], sc[mt][2 * kk2][3]);
                    pa[mt][2] = pack_bf16x2(sc[mt][2 * kk2 + 1][0], sc[mt][2 * kk2 + 1][1]);
                    pa[mt][3] = pack_bf16x2(sc[mt][2 * kk2 + 1][2], sc[mt][2 * kk2 + 1][3]);
                }
                const int key = kk2 * 16 + ((mi & 1) << 3) + l7;
#pragma unroll
                for (int nn = 0; nn < D / 16; ++nn) {
                    uint32_t v0, v1, v2, v3;
                    ldmatrix_x4_trans(vbu + tile_off(key, nn * 16 + ((mi >> 1) << 3), kPT), v0, v1, v2, v3);
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
                        mma_bf16_16816(oacc[mt][2 * nn], pa[mt], v0, v1);
                        mma_bf16_16816(oacc[mt][2 * nn + 1], pa[mt], v2, v3);
                    }
                }
            }
        }
        __syncthreads();  // every warp is done with stage s
        if (tid == 0 && i + kStages < n_tiles) {
            fence_proxy_async_smem();
            issue(i + kStages);
        }
    }

    // ---- normalise and store ------------------------------------------------------------------
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) {
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            float l = l_run[mt][h2];
            l += __shfl_xor_sync(0xffffffffu, l, 1);
            l += __shfl_xor_sync(0xffffffffu, l, 2);
            const float inv = l > 0.f ? 1.f / l : 0.f;
            if (tq[mt][h2] > t_last) continue;
            const int r = 32 * warp + 16 * mt + (lane >> 2) + 8 * h2;
            __nv_bfloat16 *orow =
                p.o + (((size_t)b * p.T + tq[mt][h2]) * p.Hq + g * p.G + r / p.QT) * D;
#pragma unroll
            for (int n = 0; n < NN; ++n)
                *reinterpret_cast<uint32_t *>(orow + n * 8 + cq) =
                    pack_bf16x2(oacc[mt][n][2 * h2] * inv, oacc[mt][n][2 * h2 + 1] * inv);
        }
    }
}

template <int D>
cudaError_t launch_d(const AttnPrefillArgs &a, cudaStream_t s) {
    constexpr int smem = smem_bytes<D>();
    const cudaError_t attr_err = once_per_device([] {
        return cudaFuncSetAttribute(attn_prefill_kernel<D>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap tmk, tmv;
    const long long n_tok = (long long)a.B * a.T;
    if (!make_tmap_tokens_sw128(&tmk, const_cast<void *>(a.k), n_tok, a.Hkv, D) ||
        !make_tmap_tokens_sw128(&tmv, const_cast<void *>(a.v), n_tok, a.Hkv, D))
        return cudaErrorInvalidValue;
    PrefillParams p;
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
    p.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    const long long grid = (long long)p.n_qb * a.B * a.Hkv;
    return launch_pdl(attn_prefill_kernel<D>, dim3((unsigned)grid), dim3(kThreads), smem, s, tmk,
                      tmv, p);
}

}  // namespace

bool attn_prefill_supported(int d, int page_tokens, int group) {
    const bool g_ok = group == 1 || group == 2 || group == 4 || group == 8 || group == 16;
    return (d == 64 || d == 128) && page_tokens == kPT && g_ok;
}

cudaError_t launch_attn_prefill(const AttnPrefillArgs &a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    if (attn_prefill_tc_supported(a.d, a.page_tokens, a.Hq / a.Hkv)) return launch_attn_prefill_tc(a, s);
    if (a.d == 128) return launch_d<128>(a, s);
    if (a.d == 64) return launch_d<64>(a, s);
    return cudaErrorInvalidValue;
}

uint32_t attn_prefill_read_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_err, sizeof v) != cudaSuccess) return 0;
    if (clear && v) {
        const unsigned int z = 0;
        cudaMemcpyToSymbol(g_err, &z, sizeof z);
    }
    return v;
}

}  // namespace hmd

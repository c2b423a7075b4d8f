// Paged split-K GQA decode attention for the FA and SWA mixers, with the new token's KV append
// fused in.
//
// FA is causal attention whose KV cache grows with the context, SWA attends to a local window
// of w keys (gist.science technical summary of "Super Apriel: One Checkpoint, Many Speeds",
// sections 1 and 2a). One decode step, per sequence b of length L (counting the new token):
//   append: write (new_k, new_v) at logical position L-1;
//   attend: o_h = softmax(q_h K^T / sqrt(d)) V over keys j in [lo, L-1], lo = 0 (FA) or
//           max(0, L - w) (SWA); query head h reads kv-head h / (Hq/Hkv).
// Paged layout: pools [n_pages][Hkv][64][d] bf16; logical page c lives at page_table[b][c] (FA)
// or at ring page page_table[b][c mod R], R = ceil(w/64) (SWA) -- a ring holding exactly the
// pages a window can touch, so logical pages map to whole ring pages.
//
// Kernel 1 (split): one CTA per work item (sequence, kv-head, key range), two resident per SM.
// The plan either fits all items in one wave of long ranges or makes about eight waves of short
// ones. A CTA streams its pages through a 3-stage TMA pipeline (two 64x64 bf16 boxes per page
// and operand, 128-byte swizzle); its 4 warps each take 16 keys of every page: S = Q K^T and O += P V run on
// mma.sync m16n8k16 (the GQA group's <=16 query heads fill the M=16 rows; tcgen05 needs M>=64),
// with an online softmax in the log2 domain. The CTA whose range holds position L-1 patches the
// new token into its shared-memory tile and writes it to the pool (the fused append). Keys
// outside [lo, L-1] are masked and their V rows zeroed in shared memory, so stale or
// uninitialised slots never reach the output. Partials (m, l, acc) go to the workspace.
// Verification (speculative decoding) is the same kernel with n_q >= 1 new tokens per sequence:
// token i sits at position P_i = L - n_q + i and attends [lo_i, P_i]; the n_q * G query rows of
// a kv-head share the MMA's 16 rows (and the one pass over the pages), each row with its own
// causal limit, and every new token is appended. n_q = 1 is the decode step.
// Kernel 2 (combine): log-sum-exp merge of the splits into bf16 o.
// The step is HBM-bound (K and V are read once: ~4 flop per byte); the design goal is to keep
// enough page copies in flight to stream at the HBM rate.
#include <cuda.h>
#include <float.h>

#include <algorithm>
#include <mutex>

#include "kernels.h"
#include "ptx.cuh"
#include "../../include/hmd.h"

namespace hmd {
namespace {

__device__ unsigned int g_err;

constexpr int kPT = 64;       // tokens per page = keys per tile
constexpr int kStages = 3;    // pages in flight per CTA
constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxGroup = 16;  // query heads per kv-head handled by one CTA (the MMA's M)
constexpr long long kWaves = 8;  // target waves of resident CTAs when ranges are split finely
constexpr long long kMaxSplits = 256;  // key ranges per (sequence, kv-head), bounds the workspace

struct SplitParams {
    const __nv_bfloat16 *q, *new_k, *new_v;
    __nv_bfloat16 *k_pool, *v_pool;
    const int32_t *page_table;
    const int32_t *seq_lens;
    const int32_t *rows;  // launch row r runs batch row rows[r] (NULL: r itself)
    float *ws_ml;   // [B*nq*Hq][n_splits][2]: running max (log2 domain), sum of exponentials
    float *ws_acc;  // [B*nq*Hq][n_splits][D]
    int B, Hq, Hkv, group, nq, n_pages, max_pages, window, swa, ring_pages;
    int n_splits, pages_per_split, max_seq_len;
    float scale_log2;  // log2(e) / sqrt(d)
    int skip_cta;      // fault injection (tests): this CTA arms its first tile with no copy
    unsigned long long wait_ns;  // limit of every bounded wait
};

// Byte offset of the 16-byte chunk holding (row, dim..dim+7) in a page tile stored as D/64
// halves of [64 rows][128 B] with the TMA 128-byte swizzle (chunk index ^= row % 8).
__device__ __forceinline__ uint32_t tile_off(int row, int dim) {
    return (uint32_t)((dim >> 6) * (kPT * 128) + row * 128 + ((((dim & 63) >> 3) ^ (row & 7)) << 4));
}

template <int D>
constexpr int stage_bytes() {
    return kStages * 2 * kPT * D * 2;
}
// stages + alignment slack (the cross-warp merge buffer reuses the stages after the last tile)
template <int D>
constexpr int smem_bytes() {
    return stage_bytes<D>() + 1024;
}

// Work item i of the split-K plan: sequence b, kv-head g, key range `split` of that sequence.
struct Item {
    int r, b, g, split, L, lo, last_page, t_begin, n_tiles;  // r: launch row, b: batch row
    bool bad_len;
};

__device__ __forceinline__ Item item_info(const SplitParams &p, int i) {
    Item it;
    it.split = i % p.n_splits;
    it.g = (i / p.n_splits) % p.Hkv;
    it.r = i / (p.n_splits * p.Hkv);
    it.b = p.rows ? p.rows[it.r] : it.r;
    it.L = p.seq_lens[it.b];
    it.bad_len = it.L < p.nq || it.L > p.max_seq_len;
    // the earliest key any row reads: that of the first new token, at position L - nq
    it.lo = (p.swa && it.L - p.nq + 1 > p.window) ? it.L - p.nq + 1 - p.window : 0;
    const int first_page = it.bad_len ? 0 : it.lo / kPT;
    it.last_page = it.bad_len ? -1 : (it.L - 1) / kPT;
    it.t_begin = first_page + it.split * p.pages_per_split;
    const int t_end = min(it.t_begin + p.pages_per_split, it.last_page + 1);
    it.n_tiles = max(0, t_end - it.t_begin);
    return it;
}

__device__ __forceinline__ int phys_page(const SplitParams &p, int b, int c) {
    const int idx = p.swa ? c % p.ring_pages : c;
    return idx < p.max_pages ? p.page_table[(size_t)b * p.max_pages + idx] : -1;
}

// Q of one (sequence, kv-head) as mma.sync A fragments: row r = i * G + j is query head
// g * G + j of new token i (rows past nq * G are zero).
template <int D>
__device__ __forceinline__ const uint32_t *q_row(const SplitParams &p, int b, int g, int r) {
    const int G = p.group;
    if (r >= p.nq * G) return nullptr;
    const int i = r / G, j = r - i * G;
    return reinterpret_cast<const uint32_t *>(p.q + (((size_t)b * p.nq + i) * p.Hq + g * G + j) * D);
}
template <int D>
__device__ __forceinline__ void load_q(const SplitParams &p, int b, int g, int lane,
                                       uint32_t (&qa)[D / 16][4]) {
    const int r0 = lane >> 2, r1 = r0 + 8, cq = (lane & 3) * 2;
    const uint32_t *q0 = q_row<D>(p, b, g, r0);
    const uint32_t *q1 = q_row<D>(p, b, g, r1);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        qa[kk][0] = q0 ? q0[(kk * 16 + cq) >> 1] : 0u;
        qa[kk][1] = q1 ? q1[(kk * 16 + cq) >> 1] : 0u;
        qa[kk][2] = q0 ? q0[(kk * 16 + 8 + cq) >> 1] : 0u;
        qa[kk][3] = q1 ? q1[(kk * 16 + 8 + cq) >> 1] : 0u;
    }
}

// Split-K kernel: CTA i processes work item i. Warp 0 produces: its lanes hold the physical
// pages of 32 consecutive tiles (one coalesced page-table load per 32 tiles, fetched a chunk
// ahead), and lane 0 issues each tile's TMA copies and records the tile's page in shared memory
// before arming the stage's barrier. The tile loop itself reads no global memory.
template <int D>
__global__ void __launch_bounds__(kThreads, 2)
attn_split_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                  const SplitParams p) {
    constexpr int TB = kPT * D * 2;  // bytes of one page of one head (K or V)
    constexpr int NK = D / 16;       // k-steps of Q K^T
    constexpr int NN = D / 8;        // n-tiles of P V
    constexpr int RS = D + 2;
    static_assert(kWarps * kMaxGroup * RS * 4 <= stage_bytes<D>(), "merge buffer fits the stages");
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ int stage_pg[kStages];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const uint32_t smem_base = smem_u32(smem);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = p.group;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&full_bar[s]), 1);
        fence_barrier_init();
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    griddep_launch_dependents();
    griddep_wait();  // q, the new token, the pools and the tables may come from the previous kernel
    const Item it = item_info(p, blockIdx.x);
    if (tid == 0 && it.bad_len && it.split == 0) atomicOr(&g_err, HMD_DEVERR_SEQLEN);

    // ---- producer (warp 0, warp-uniform calls; lane 0 issues) -----------------------------
    auto table_entry = [&](int t) -> int {
        return t < it.n_tiles ? phys_page(p, it.b, it.t_begin + t) : -1;
    };
    int pt_cur = -1, pt_next = -1, issued = 0;
    if (warp == 0) {
        pt_cur = table_entry(lane);
        pt_next = table_entry(32 + lane);
    }
    auto issue_next = [&]() {
        if (issued >= it.n_tiles) return;
        if (issued > 0 && (issued & 31) == 0) {
            pt_cur = pt_next;
            pt_next = table_entry(issued + 32 + lane);
        }
        const int pg = __shfl_sync(0xffffffffu, pt_cur, issued & 31);
        if (lane == 0) {
            const int s = issued % kStages;
            const uint32_t bar = smem_u32(&full_bar[s]);
            if (pg < 0 || pg >= p.n_pages) {
                stage_pg[s] = -1;
                atomicOr(&g_err, HMD_DEVERR_PAGE);
                mbar_arrive_expect_tx(bar, 0);  // complete the phase with no copy
            } else {
                stage_pg[s] = pg;
                mbar_arrive_expect_tx(bar, 2 * TB);
                const uint32_t kb = smem_base + s * 2 * TB, vb = kb + TB;
                const int y = (pg * p.Hkv + it.g) * kPT;
                // a test may arm the first tile's barrier with no copy
                if (issued > 0 || (int)blockIdx.x != p.skip_cta) {
#pragma unroll
                    for (int hf = 0; hf < D / 64; ++hf) {
                        tma_load_2d(kb + hf * kPT * 128, &tmk, bar, hf * 64, y);
                        tma_load_2d(vb + hf * kPT * 128, &tmv, bar, hf * 64, y);
                    }
                }
            }
        }
        ++issued;
    };
    __syncthreads();  // barriers initialised
    if (warp == 0) {
        for (int t = 0; t < kStages; ++t) issue_next();
    }

    const int r0 = lane >> 2, r1 = r0 + 8, cq = (lane & 3) * 2, mi = lane >> 3;
    uint32_t qa[NK][4];
    load_q<D>(p, it.b, it.g, lane, qa);
    // keys [lo_r, hi_r] of this thread's two rows (token r / G sits at L - nq + r / G); rows past
    // nq * G read nothing
    const int rows = p.nq * G, first_new = it.L - p.nq;
    int row_lo[2], row_hi[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int r = rr ? r1 : r0;
        row_hi[rr] = r < rows ? first_new + r / G : -1;
        row_lo[rr] = (p.swa && row_hi[rr] + 1 > p.window) ? row_hi[rr] + 1 - p.window : 0;
    }
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    float oacc[NN][4];
#pragma unroll
    for (int n = 0; n < NN; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;

    for (int t = 0; t < it.n_tiles; ++t) {
        const int s = t % kStages;
        const bool ok = mbar_wait_bounded(smem_u32(&full_bar[s]), (t / kStages) & 1, p.wait_ns);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
                // let the copies this CTA issued finish (bounded) before leaving
                for (int u = t; u < issued; ++u)
                    (void)mbar_wait_bounded(smem_u32(&full_bar[u % kStages]), (u / kStages) & 1,
                                            p.wait_ns);
            }
            // mark this range's partials as missing (a negative sum of exponentials, which no
            // completed range writes): the combine then leaves these rows' outputs untouched
            for (int r = tid; r < p.nq * G; r += kThreads) {
                const int ti = r / G;
                const size_t row = (((size_t)it.r * p.nq + ti) * p.Hq + it.g * G + (r - ti * G)) *
                                       p.n_splits + it.split;
                p.ws_ml[row * 2 + 1] = -1.f;
            }
            return;  // the error word reports the step as failed
        }
        const int pg = stage_pg[s];
        const bool tile_ok = pg >= 0;
        const int c = it.t_begin + t;
        const int base = c * kPT;
        uint8_t *kb = smem + s * 2 * TB;
        uint8_t *vb = kb + TB;
        const bool has_new = base <= it.L - 1 && base + kPT - 1 >= first_new;
        const bool partial = base < it.lo || base + kPT - 1 > it.L - 1;
        if (tile_ok && (has_new || partial)) {
            // zero V rows of masked positions; patch in the new token's K and V
            for (int idx = tid; idx < kPT * (D / 8); idx += kThreads) {
                const int row = idx / (D / 8), ch = idx % (D / 8);
                const int pos = base + row;
                if (pos < it.lo || pos > it.L - 1)
                    *reinterpret_cast<uint4 *>(vb + tile_off(row, ch * 8)) = make_uint4(0, 0, 0, 0);
            }
            if (has_new) {
                for (int idx = tid; idx < p.nq * 2 * (D / 8); idx += kThreads) {
                    const int i = idx / (2 * (D / 8)), ch = idx - i * (2 * (D / 8));
                    const int pos = first_new + i;
                    if (pos < base || pos >= base + kPT) continue;  // token i is in another tile
                    const int rr = pos - base;
                    const size_t src = (((size_t)it.b * p.nq + i) * p.Hkv + it.g) * D;
                    const int cc = ch % (D / 8);
                    const uint4 val = ch < D / 8
                        ? *reinterpret_cast<const uint4 *>(p.new_k + src + cc * 8)
                        : *reinterpret_cast<const uint4 *>(p.new_v + src + cc * 8);
                    uint8_t *dst = (ch < D / 8 ? kb : vb) + tile_off(rr, cc * 8);
                    *reinterpret_cast<uint4 *>(dst) = val;
                    // the append itself: the pool slot of position L - nq + i
                    __nv_bfloat16 *pool = ch < D / 8 ? p.k_pool : p.v_pool;
                    *reinterpret_cast<uint4 *>(pool + (((size_t)pg * p.Hkv + it.g) * kPT + rr) * D + cc * 8) = val;
                }
            }
            fence_proxy_async_smem();  // these generic writes precede the stage's next TMA fill
            __syncthreads();
        }

        if (tile_ok) {
            const uint32_t kbu = smem_u32(kb), vbu = smem_u32(vb);
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            {
                const int key = warp * 16 + ((mi >> 1) << 3) + (lane & 7);
#pragma unroll
                for (int kk = 0; kk < NK; ++kk) {
                    uint32_t b00, b01, b10, b11;
                    ldmatrix_x4(kbu + tile_off(key, kk * 16 + ((mi & 1) << 3)), b00, b01, b10, b11);
                    mma_bf16_16816(sc[0], qa[kk], b00, b01);
                    mma_bf16_16816(sc[1], qa[kk], b10, b11);
                }
            }
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 2; ++j) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int pos = base + warp * 16 + j * 8 + cq + (e & 1);
                    const bool valid = pos >= row_lo[e >> 1] && pos <= row_hi[e >> 1];
                    sc[j][e] = valid ? sc[j][e] * p.scale_log2 : -INFINITY;
                    mx[e >> 1] = fmaxf(mx[e >> 1], sc[j][e]);
                }
            }
            float corr[2], mu[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
                const float mnew = fmaxf(m_run[r], mx[r]);
                mu[r] = (mnew == -INFINITY) ? 0.f : mnew;
                corr[r] = exp2f(m_run[r] - mu[r]);
                m_run[r] = mnew;
            }
            float ls[2] = {0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 2; ++j) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    sc[j][e] = exp2f(sc[j][e] - mu[e >> 1]);
                    ls[e >> 1] += sc[j][e];
                }
            }
            l_run[0] = l_run[0] * corr[0] + ls[0];
            l_run[1] = l_run[1] * corr[1] + ls[1];
#pragma unroll
            for (int n = 0; n < NN; ++n) {
                oacc[n][0] *= corr[0]; oacc[n][1] *= corr[0];
                oacc[n][2] *= corr[1]; oacc[n][3] *= corr[1];
            }
            uint32_t pa[4];
            pa[0] = pack_bf16x2(sc[0][0], sc[0][1]);
            pa[1] = pack_bf16x2(sc[0][2], sc[0][3]);
            pa[2] = pack_bf16x2(sc[1][0], sc[1][1]);
            pa[3] = pack_bf16x2(sc[1][2], sc[1][3]);
            {
                const int key = warp * 16 + ((mi & 1) << 3) + (lane & 7);
#pragma unroll
                for (int nn = 0; nn < D / 16; ++nn) {
                    uint32_t v0, v1, v2, v3;
                    ldmatrix_x4_trans(vbu + tile_off(key, nn * 16 + ((mi >> 1) << 3)), v0, v1, v2, v3);
                    mma_bf16_16816(oacc[2 * nn], pa, v0, v1);
                    mma_bf16_16816(oacc[2 * nn + 1], pa, v2, v3);
                }
            }
        }
        __syncthreads();  // every warp is done with stage s
        if (warp == 0) {
            if (lane == 0) fence_proxy_async_smem();
            issue_next();
        }
    }

    // ---- merge the 4 warps' partials (the stages are idle now: reuse them) -------------------
    float *red = reinterpret_cast<float *>(smem);  // [kWarps][rows][D + 2]
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        float l = l_run[r];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        l_run[r] = l;
    }
    if (r0 < rows) {
        float *dst = red + (warp * rows + r0) * RS;
#pragma unroll
        for (int n = 0; n < NN; ++n) {
            dst[n * 8 + cq] = oacc[n][0];
            dst[n * 8 + cq + 1] = oacc[n][1];
        }
        if ((lane & 3) == 0) { dst[D] = m_run[0]; dst[D + 1] = l_run[0]; }
    }
    if (r1 < rows) {
        float *dst = red + (warp * rows + r1) * RS;
#pragma unroll
        for (int n = 0; n < NN; ++n) {
            dst[n * 8 + cq] = oacc[n][2];
            dst[n * 8 + cq + 1] = oacc[n][3];
        }
        if ((lane & 3) == 0) { dst[D] = m_run[1]; dst[D + 1] = l_run[1]; }
    }
    __syncthreads();
    for (int idx = tid; idx < rows * D; idx += kThreads) {
        const int r = idx / D, dim = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red[(w * rows + r) * RS + D]);
        float acc = 0.f, lsum = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float f = exp2f(red[(w * rows + r) * RS + D] - M);
                acc += f * red[(w * rows + r) * RS + dim];
                lsum += f * red[(w * rows + r) * RS + D + 1];
            }
        }
        const int ti = r / G;  // new token ti, query head g * G + (r - ti * G)
        const size_t row = (((size_t)it.r * p.nq + ti) * p.Hq + it.g * G + (r - ti * G)) * p.n_splits + it.split;
        p.ws_acc[row * D + dim] = acc;
        if (dim == 0) {
            p.ws_ml[row * 2] = M;
            p.ws_ml[row * 2 + 1] = lsum;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(D) attn_combine_kernel(const float *ws_ml, const float *ws_acc,
                                                         int n_splits, __nv_bfloat16 *o,
                                                         const int32_t *rows, int per_row) {
    const size_t bh = blockIdx.x;  // query row of the launch: (launch row, token, head)
    const int dim = threadIdx.x;
    griddep_launch_dependents();
    griddep_wait();  // the partials are the split kernel's output
    const size_t ob = rows ? (size_t)rows[bh / per_row] * per_row + bh % per_row : bh;
    const float *ml = ws_ml + bh * n_splits * 2;
    float M = -INFINITY;
    bool missing = false;  // a key range whose CTA gave up (see the split kernel's abort path)
    for (int s = 0; s < n_splits; ++s) {
        M = fmaxf(M, ml[2 * s]);
        missing |= ml[2 * s + 1] < 0.f;
    }
    if (missing) return;
    float num = 0.f, den = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < n_splits; ++s) {
            const float f = exp2f(ml[2 * s] - M);
            num += f * ws_acc[(bh * n_splits + s) * D + dim];
            den += f * ml[2 * s + 1];
        }
    }
    o[ob * D + dim] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
}

// ---- host side --------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Tensor map over a pool viewed as [n_pages*Hkv*64 rows][d] bf16, box 64x64, 128-byte swizzle.
bool make_pool_map(CUtensorMap *m, void *pool, int n_pages, int Hkv, int d) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)d, (cuuint64_t)n_pages * Hkv * kPT};
    const cuuint64_t gstride[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kPT};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pool, gdim, gstride, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const AttnDecodeArgs &a, const AttnPlan &plan, cudaStream_t s) {
    const int group = a.Hq / a.Hkv;
    constexpr int smem = smem_bytes<D>();
    const cudaError_t attr_err = once_per_device([] {
        return cudaFuncSetAttribute(attn_split_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    smem_bytes<D>());
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap tmk, tmv;
    if (!make_pool_map(&tmk, a.k_pool, a.n_pages, a.Hkv, D) ||
        !make_pool_map(&tmv, a.v_pool, a.n_pages, a.Hkv, D))
        return cudaErrorInvalidValue;
    SplitParams p;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.new_k = static_cast<const __nv_bfloat16 *>(a.new_k);
    p.new_v = static_cast<const __nv_bfloat16 *>(a.new_v);
    p.k_pool = static_cast<__nv_bfloat16 *>(a.k_pool);
    p.v_pool = static_cast<__nv_bfloat16 *>(a.v_pool);
    p.page_table = a.page_table;
    p.seq_lens = a.seq_lens;
    p.rows = a.rows;
    const int n_run = a.rows ? a.n_rows : a.B;  // batch rows this launch runs
    const size_t rows = (size_t)n_run * a.nq * a.Hq * plan.n_splits;
    p.ws_ml = static_cast<float *>(a.workspace);
    p.ws_acc = p.ws_ml + ((rows * 2 + 3) & ~static_cast<size_t>(3));
    p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.group = group; p.nq = a.nq;
    p.n_pages = a.n_pages; p.max_pages = a.max_pages;
    p.window = a.window; p.swa = a.swa ? 1 : 0;
    p.ring_pages = a.swa ? a.ring_pages : 0;
    p.n_splits = plan.n_splits; p.pages_per_split = plan.pages_per_split;
    p.max_seq_len = a.max_seq_len;
    p.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    p.skip_cta = a.skip.cta;
    p.wait_ns = a.skip.wait_ns;
    cudaError_t e = launch_pdl(attn_split_kernel<D>, dim3((unsigned)plan.n_ctas), dim3(kThreads),
                               smem, s, tmk, tmv, p);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_combine_kernel<D>, dim3((unsigned)(n_run * a.nq * a.Hq)), dim3(D), 0, s,
                      (const float *)p.ws_ml, (const float *)p.ws_acc, plan.n_splits,
                      static_cast<__nv_bfloat16 *>(a.o), a.rows, a.nq * a.Hq);
}

// SMs of the current device (148 when no device can be queried).
int device_sms() {
    return once_per_device([] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            return v;
        cudaGetLastError();
        return 148;
    });
}

}  // namespace

bool attn_decode_supported(int d, int page_tokens, int group, int nq) {
    return (d == 64 || d == 128) && page_tokens == kPT && group >= 1 && nq >= 1 &&
           (long long)group * nq <= kMaxGroup;
}

AttnPlan attn_decode_plan(bool swa, int window, int B, int Hq, int Hkv, int d, int page_tokens,
                          int max_seq_len, int nq) {
    (void)page_tokens;
    (void)Hq;
    AttnPlan pl;
    long long tiles = (max_seq_len + kPT - 1) / kPT;
    if (swa) tiles = std::min<long long>(tiles, ((long long)window + nq - 1 + kPT - 1) / kPT + 1);
    tiles = std::max<long long>(tiles, 1);
    const long long units = std::max<long long>(1, (long long)B * Hkv);
    // resident CTAs per SM from shared memory (228 KiB per SM, 1 KiB reserved per CTA)
    const int smem = (d == 64 ? smem_bytes<64>() : smem_bytes<128>()) + 1024;
    const long long slots = (long long)std::max(1, std::min(2, 233472 / smem)) * device_sms();
    // One wave: the most key ranges that still fit every item in a resident slot, so each CTA
    // streams one long range. Taken when it fills at least 3/4 of the slots; otherwise about
    // kWaves waves of shorter ranges (>= 2 pages each), which the block scheduler balances.
    long long s_one = std::max<long long>(1, std::min({tiles, slots / units, kMaxSplits}));
    long long s_many = std::max<long long>(
        1, std::min({(kWaves * slots + units - 1) / units, std::max<long long>(1, tiles / 2),
                     kMaxSplits}));
    const bool one_wave_fits = units * s_one <= slots && units * s_one * 4 >= slots * 3;
    long long splits = (one_wave_fits || units * s_many <= slots) ? s_one : s_many;
    const long long pps = (tiles + splits - 1) / splits;
    splits = (tiles + pps - 1) / pps;  // no empty range
    pl.n_splits = (int)splits;
    pl.pages_per_split = (int)pps;
    pl.n_ctas = (int)(units * splits);
    const size_t rows = (size_t)B * nq * Hq * splits;
    pl.ws_bytes = (((rows * 2 + 3) & ~static_cast<size_t>(3)) + rows * d) * sizeof(float);
    return pl;
}

cudaError_t launch_attn_decode(const AttnDecodeArgs &a, cudaStream_t s) {
    const AttnPlan plan = attn_decode_plan(a.swa, a.window, a.rows ? a.n_rows : a.B, a.Hq, a.Hkv,
                                           a.d, a.page_tokens, a.max_seq_len, a.nq);
    if (a.d == 128) return launch_d<128>(a, plan, s);
    if (a.d == 64) return launch_d<64>(a, plan, s);
    return cudaErrorInvalidValue;
}

uint32_t attn_decode_read_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_err, sizeof v) != cudaSuccess) return 0;
    if (clear && v) {
        const unsigned int z = 0;
        cudaMemcpyToSymbol(g_err, &z, sizeof z);
    }
    return v;
}

}  // namespace hmd

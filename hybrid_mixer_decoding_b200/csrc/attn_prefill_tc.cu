// FA / SWA prefill on the 5th-generation tensor cores (tcgen05, TMEM), d = 64 or 128.
//
// FA and SWA from the gist.science technical summary of "Super Apriel: One Checkpoint, Many
// Speeds", sections 1 and 2a: token t of a prompt attends keys [lo_t, t], lo_t = 0 (FA) or
// max(0, t + 1 - w) (SWA), and the prompt's K and V are written to the paged cache at the slots
// the decode step reads (SWA: the positions the ring of ceil(w / 64) pages keeps).
//
// One CTA per (sequence, kv-head, block of 256/G tokens): two query tiles of 128 rows (row r of
// tile j: head g*G + r / QT, token t_first + j*QT + r % QT, QT = 128/G) share every K/V tile.
// Key tiles of 128. Warp-specialised, 320 threads:
//   warp 9 (one lane) streams K and V tiles by TMA into two rings of two stages (3-D boxes of
//     64 prompt tokens, or 2-D boxes of one cache page, 128-byte swizzle);
//   warp 8 (one lane) issues the tcgen05.mma products, per key tile i and query tile j:
//       S_j = Q_j K_i^T   M=128 N=128 K=d (both from shared memory, K-major) into TMEM S_j
//       O_j += P_j V_i    M=128 N=d K=128 (P_j from TMEM, V MN-major from shared memory)
//     in the order O_0(i), S_0(i+1), O_1(i), S_1(i+1): while one query tile's softmax runs, the
//     tensor core works on the other's products;
//   warps 4j .. 4j+3 are query tile j's softmax group: thread = query row = TMEM lane. A thread
//     reads its row of S_j (tcgen05.ld), takes the maximum itself (no exchange), writes the
//     row of P_j (bf16 pairs) into the TMEM columns of S_j it has read (tcgen05.st), and hands
//     over through an mbarrier.
// P_j (128 keys as bf16 pairs) lies in the first 64 columns of S_j: S_j(i+1) is issued after
// O_j(i) by the same thread, and the tensor core runs one thread's products in order.
// Lazy rescaling, per row: O_j accumulates at a fixed exponent base per row, which moves only
// when the row's maximum exceeds it by more than 8 (P stays below 2^8); the thread then scales
// its row of O_j in TMEM. S_j(i) is issued after O_j(i-1), so once S_j(i) is complete the
// previous product into O_j is too, and the row can be rescaled before O_j(i) is issued.
// Every wait is bounded; a wait that gives up raises a shared abort flag that ends every other
// wait of the CTA, and the error word reports the call as failed.
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

constexpr int kPT = 64;          // tokens per page = keys per TMA box
constexpr int kKT = 128;         // keys per tile
constexpr int kRows = 128;       // rows per query tile
constexpr int kSoftmax = 256;    // softmax threads (warps 0-7: two groups of four)
constexpr int kThreads = kSoftmax + 64;  // + the MMA warp (8) and the TMA warp (9)
constexpr uint32_t kTmemCols = 512;  // query tile j: S_j (and P_j) at 256 j, O_j at 256 j + 128

// shared memory (bytes from a 1024-aligned base) for head size D (64 or 128). Every operand tile
// is stored as D / 64 blocks of [128 rows][128 B] with the 128-byte swizzle; a K or V tile's
// rows are its 128 keys, the two 64-key boxes at +0 and +8 KiB of each block.
template <int D>
struct Smem {
    static constexpr uint32_t BLK = kRows * 128;               // one [128 rows][128 B] block
    static constexpr uint32_t TILE = (D / 64) * BLK;           // a query tile, a K or a V stage
    static constexpr uint32_t OFF_Q = 0;                       // Q_0, Q_1
    static constexpr uint32_t OFF_K = OFF_Q + 2 * TILE;        // K stages 0, 1
    static constexpr uint32_t OFF_V = OFF_K + 2 * TILE;        // V stages 0, 1
    static constexpr uint32_t OFF_BAR = OFF_V + 2 * TILE;
    static constexpr uint32_t USED = OFF_BAR + 256 + 1024;
    // at least 116 KiB, so that one CTA (and its 512 TMEM columns) holds an SM
    static constexpr uint32_t BYTES = USED > 118784 ? USED : 118784;
};
static_assert(Smem<128>::BYTES <= 232448, "shared memory per CTA");
static_assert(2 * Smem<64>::BYTES > 233472, "one CTA per SM");
// barrier indices
constexpr int B_KFULL = 0;   // [2] K tile landed (TMA)
constexpr int B_VFULL = 2;   // [2] V tile landed (TMA)
constexpr int B_KFREE = 4;   // [2] both S products of the K tile done (commit)
constexpr int B_VFREE = 6;   // [2] both PV products of the V tile done (commit)
constexpr int B_SFULL = 8;   // [2] per query tile: S_j computed (commit)
constexpr int B_PFULL = 10;  // [2] per query tile: P_j written (four warps)
constexpr int B_ODONE = 12;  // [2] per query tile: the last PV product done (commit)
constexpr int B_FINAL = 14;  // every product issued done (commit, teardown)
constexpr int N_BARS = 15;
constexpr float kLazy = 8.f;  // log2 headroom before a row's exponent base moves

constexpr uint32_t ID_S = idesc_bf16(128, kKT, 0, 0);   // A = Q (K-major), B = K (K-major)
template <int D>
constexpr uint32_t ID_PV = idesc_bf16(128, D, 0, 1);     // A = P (TMEM), B = V (MN-major)

// ---- two fp32 lanes per instruction (sm_100 f32x2 arithmetic) ----------------------------------
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x for two lanes on the FMA pipe, for x <= 8: 2^x = 2^n 2^f with n = x rounded to the
// nearest integer (adding 1.5 * 2^23 rounds it into the low mantissa bits) and f = x - n in
// [-1/2, 1/2], 2^f by a cubic fitted to it on that interval (iteratively reweighted least
// squares at Chebyshev nodes; largest relative error 7.5e-5, far below the bf16 rounding of P).
// n is added to the exponent field straight from the rounded sum's bits (its low bits hold n,
// the bits above them drop out of the shift). x is clamped at -125, where 2^x is below 1e-37
// and its share of a row sum that holds an entry >= 1 is nil. Splitting the exponentials
// between this and ex2.approx keeps the softmax off a single pipe.
__device__ __forceinline__ uint64_t exp2_fma_x2(uint64_t x2) {
    float a, b;
    f2_split(x2, a, b);
    x2 = f2(fmaxf(a, -125.f), fmaxf(b, -125.f));
    const uint64_t j = f2_add(x2, f2(12582912.f, 12582912.f));
    const uint64_t n = f2_add(j, f2(-12582912.f, -12582912.f));
    const uint64_t f = f2_fma(n, f2(-1.f, -1.f), x2);
    uint64_t p = f2_fma(f2(0.05517588f, 0.05517588f), f, f2(0.24261151f, 0.24261151f));
    p = f2_fma(p, f, f2(0.6932602f, 0.6932602f));
    p = f2_fma(p, f, f2(0.999928f, 0.999928f));
    float p0, p1, j0, j1;
    f2_split(p, p0, p1);
    f2_split(j, j0, j1);
    return f2(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(j0) << 23)),
              __uint_as_float(__float_as_uint(p1) + (__float_as_uint(j1) << 23)));
}

struct TcParams {
    const __nv_bfloat16 *q, *k, *v;
    __nv_bfloat16 *k_pool, *v_pool, *o;
    const int32_t *page_table;
    const int32_t *prefix_lens;  // cached positions before the prompt, per sequence (or NULL)
    int B, T, Hq, Hkv, G, QT, n_qb;
    int window, swa, ring_pages, max_pages, n_pages;
    int defer_write;  // the prompt's K/V go to the cache in a later kernel (SWA with a prefix)
    float scale_log2;
};

// byte offset of (row, col..col+7) in [rows][128 B] blocks of 64 columns, 128-byte swizzle
__device__ __forceinline__ uint32_t swz(int row, int col, int rows) {
    return (uint32_t)((col >> 6) * rows * 128 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4));
}

__device__ __forceinline__ int key_lo(const TcParams &p, int t) {
    return (p.swa && t + 1 > p.window) ? t + 1 - p.window : 0;
}

// Bounded wait that also gives up as soon as another thread of the CTA raised `abort`.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            return false;
        }
    }
}

// PREFIX: sequences may start after cached positions (p.prefix_lens); false compiles the
// empty-cache prefill with every prefix path removed. D: head size, 64 or 128.
template <int D, bool PREFIX>
__global__ void __launch_bounds__(kThreads, 1)
attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                       const __grid_constant__ CUtensorMap tmpk,
                       const __grid_constant__ CUtensorMap tmpv, const TcParams p) {
    using L = Smem<D>;
    constexpr uint32_t OFF_Q = L::OFF_Q, OFF_K = L::OFF_K, OFF_V = L::OFF_V, TILE = L::TILE,
                       OFF_BAR = L::OFF_BAR, BLK = L::BLK;
    constexpr int kD = D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 8 * N_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_BAR + 8 * N_BARS + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int bg = blockIdx.x % (p.B * p.Hkv);
    const int qb = p.n_qb - 1 - (int)(blockIdx.x / (p.B * p.Hkv));  // longest blocks first
    const int b = bg / p.Hkv, g = bg - b * p.Hkv;
    const int t_first = qb * 2 * p.QT;
    const int t_last = min(p.T, t_first + 2 * p.QT) - 1;

    if (tid == 0) {
        for (int i = 0; i < N_BARS; ++i) mbar_init(bar(i), (i == B_PFULL || i == B_PFULL + 1) ? 4 : 1);
        fence_barrier_init();
        *abort_flag = 0;
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        if constexpr (PREFIX) {
            prefetch_tmap(&tmpk);
            prefetch_tmap(&tmpv);
        }
    }
    if (warp == 8) {
        __syncwarp();  // tcgen05.alloc is .sync.aligned: the whole warp, converged
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    griddep_launch_dependents();
    griddep_wait();  // the prompt and the cache may come from the previous kernel

    // positions: token t of the prompt sits at L0 + t after a cached prefix of L0 positions
    int L0 = 0;
    if constexpr (PREFIX) {
        L0 = p.prefix_lens[b];
        if (L0 < 0 || (L0 % kPT) != 0) {  // not a whole number of pages: report, run without it
            if (tid == 0) atomicOr(&g_err, HMD_DEVERR_SEQLEN);
            L0 = 0;
        }
    }
    const int kb_lo = key_lo(p, L0 + t_first) / kKT, kb_hi = (L0 + t_last) / kKT;
    const int n_tiles = kb_hi - kb_lo + 1;

    // ---- Q rows -> shared memory (one row per softmax thread); fused cache write -------------
    const int qt = warp >> 2;  // the softmax thread's query tile
    const int row = tid & (kRows - 1);
    const int t_row = t_first + qt * p.QT + row % p.QT;
    const bool row_ok = t_row <= t_last;
    const int pos_row = L0 + t_row;  // the row's position: its last key
    const int lo_row = key_lo(p, pos_row);
    const int h_row = g * p.G + row / p.QT;
    if (tid < kSoftmax) {
        const uint4 *src = reinterpret_cast<const uint4 *>(
            p.q + (((size_t)b * p.T + (row_ok ? t_row : 0)) * p.Hq + h_row) * kD);
#pragma unroll
        for (int c = 0; c < kD / 8; ++c) {
            const uint4 v = row_ok ? src[c] : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sm + OFF_Q + qt * TILE + swz(row, c * 8, kRows)) = v;
        }
        const int ring = p.ring_pages * kPT;
        const int n_tok = t_last - t_first + 1;
        constexpr int CH = kD / 8;
        for (int idx = tid; idx < ((PREFIX && p.defer_write) ? 0 : n_tok * 2 * CH); idx += kSoftmax) {
            const int tt = idx / (2 * CH), rem = idx - tt * 2 * CH;
            const bool is_v = rem >= CH;
            const int chk = is_v ? rem - CH : rem;
            const int t = t_first + tt;
            if (p.swa && t < p.T - ring) continue;  // overwritten later in the ring
            const int li = p.swa ? (L0 + t) % ring : L0 + t;
            const int lp = li / kPT;
            const int pg = lp < p.max_pages ? p.page_table[(size_t)b * p.max_pages + lp] : -1;
            if (pg < 0 || pg >= p.n_pages) {
                atomicOr(&g_err, HMD_DEVERR_PAGE);
                continue;
            }
            const size_t srco = (((size_t)b * p.T + t) * p.Hkv + g) * kD + chk * 8;
            const size_t dsto = (((size_t)pg * p.Hkv + g) * kPT + (li % kPT)) * kD + chk * 8;
            *reinterpret_cast<uint4 *>((is_v ? p.v_pool : p.k_pool) + dsto) =
                *reinterpret_cast<const uint4 *>((is_v ? p.v : p.k) + srco);
        }
        fence_proxy_async_smem();  // Q is read by the tensor cores
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 9) {
        // ================= TMA producer (one lane) ======================================
        if (lane == 0) {
            int issued = 0;  // K/V tiles issued
            // K or V of tile i into stage i % 2: two boxes of 64 keys (a page of the cached
            // prefix, or 64 prompt tokens; boxes past the prompt's end read zeros or another
            // sequence's rows, masked by every row)
            auto issue_kv = [&](int i, bool is_v) {
                const int st = i & 1;
                const uint32_t dst = sb + (is_v ? OFF_V : OFF_K) + st * TILE;
                const uint32_t fb = bar((is_v ? B_VFULL : B_KFULL) + st);
                const CUtensorMap *tm = is_v ? &tmv : &tmk;
                int pg2[2] = {-1, -1};
                uint32_t bytes = 0;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int key0 = (kb_lo + i) * kKT + h * kPT;  // first position of the box
                    if (PREFIX && key0 < L0) {
                        const int lp = (key0 / kPT) % (p.swa ? p.ring_pages : 0x7fffffff);
                        const int pg = lp < p.max_pages ? p.page_table[(size_t)b * p.max_pages + lp] : -1;
                        if (pg < 0 || pg >= p.n_pages) {
                            atomicOr(&g_err, HMD_DEVERR_PAGE);
                            continue;  // no copy: the call reports the error
                        }
                        pg2[h] = pg;
                    }
                    bytes += (kD / 64) * 8192;
                }
                mbar_arrive_expect_tx(fb, bytes);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int key0 = (kb_lo + i) * kKT + h * kPT;
                    if (PREFIX && key0 < L0) {
                        if (pg2[h] < 0) continue;
                        const int y = (pg2[h] * p.Hkv + g) * kPT;
#pragma unroll
                        for (int hf = 0; hf < kD / 64; ++hf)
                            tma_load_2d(dst + hf * BLK + h * 8192, is_v ? &tmpv : &tmpk, fb, hf * 64, y);
                    } else {
                        const int z = b * p.T + (key0 - L0);
#pragma unroll
                        for (int hf = 0; hf < kD / 64; ++hf)
                            tma_load_3d(dst + hf * BLK + h * 8192, tm, fb, hf * 64, g, z);
                    }
                }
            };
            bool ok = true;
            for (int t = 0; t < n_tiles && ok; ++t) {
                const int st = t & 1;
                if (t >= 2) ok = wait_or_abort(bar(B_KFREE + st), ((t - 2) >> 1) & 1, abort_flag);
                if (!ok) break;
                issue_kv(t, false);
                if (t >= 2) ok = wait_or_abort(bar(B_VFREE + st), ((t - 2) >> 1) & 1, abort_flag);
                if (!ok) {
                    issued = 2 * t + 1;
                    break;
                }
                issue_kv(t, true);
                issued = 2 * t + 2;
            }
            if (!ok) {
                // the copies in flight land (bounded) before shared memory is released
                atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
                for (int u = max(0, issued - 4); u < issued; ++u) {
                    const int t = u >> 1;
                    (void)mbar_wait_bounded(bar(((u & 1) ? B_VFULL : B_KFULL) + (t & 1)), (t >> 1) & 1);
                }
            }
        }
    } else if (warp == 8) {
        // ================= MMA issue (one lane) ========================================
        if (lane == 0) {
            // descriptors: the address field is the byte address / 16, so an offset is added as
            // offset / 16 (every address here is below 256 KiB: no carry out of the field)
            const uint64_t d_q = smem_desc_sw128(sb + OFF_Q, 16, 1024);
            const uint64_t d_k = smem_desc_sw128(sb + OFF_K, 16, 1024);
            const uint64_t d_v = smem_desc_sw128(sb + OFF_V, BLK, 1024);
            auto issue_s = [&](int j, int i) {  // S_j = Q_j K_i^T
                const uint64_t qo = (j * TILE) >> 4, ko = ((i & 1) * TILE) >> 4;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * BLK + (kk & 3) * 32;
                    umma_bf16(tmem + 256 * j, d_q + qo + (off >> 4), d_k + ko + (off >> 4), ID_S, kk > 0);
                }
                umma_commit(bar(B_SFULL + j));
            };
            auto issue_pv = [&](int j, int i) {  // O_j (+)= P_j V_i, P_j from TMEM
                const uint64_t vo = ((i & 1) * TILE) >> 4;
#pragma unroll
                for (int kk = 0; kk < kKT / 16; ++kk)
                    umma_bf16_ts(tmem + 256 * j + 128, tmem + 256 * j + 8 * kk, d_v + vo + ((kk * 2048) >> 4),
                                 ID_PV<kD>, (i > 0 || kk > 0) ? 1u : 0u);
            };
            bool ok = wait_or_abort(bar(B_KFULL), 0, abort_flag);
            bool issued_any = false;
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(1, 0);
                umma_commit(bar(B_KFREE));
                issued_any = true;
            }
            for (int i = 0; i < n_tiles && ok; ++i) {
#pragma unroll 1
                for (int j = 0; j < 2 && ok; ++j) {
                    ok = wait_or_abort(bar(B_PFULL + j), i & 1, abort_flag);
                    if (ok && j == 0) ok = wait_or_abort(bar(B_VFULL + (i & 1)), (i >> 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(j, i);
                    if (j == 1) umma_commit(bar(B_VFREE + (i & 1)));
                    if (i == n_tiles - 1) umma_commit(bar(B_ODONE + j));
                    if (i + 1 < n_tiles) {
                        if (j == 0)
                            ok = wait_or_abort(bar(B_KFULL + ((i + 1) & 1)), ((i + 1) >> 1) & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(j, i + 1);
                        if (j == 1) umma_commit(bar(B_KFREE + ((i + 1) & 1)));
                    }
                }
            }
            if (!ok) atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
            if (issued_any) {
                // every product this thread issued is done before TMEM is freed (bounded)
                umma_commit(bar(B_FINAL));
                (void)mbar_wait_bounded(bar(B_FINAL), 0);
            }
        }
    } else {
        // ================= softmax: query tile qt, one thread per row ======================
        const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const uint32_t s_col = lane_base + 256 * qt, o_col = s_col + 128;
        float m_base = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int i = 0; i < n_tiles && ok; ++i) {
            ok = wait_or_abort(bar(B_SFULL + qt), i & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);  // the TMEM accesses below run converged
            if (!ok) break;
            tc_fence_after();
            float s[kKT];
            {
                uint32_t r[64];
                tmem_ld64(s_col, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 64; ++j) s[j] = __uint_as_float(r[j]);
                tmem_ld64(s_col + 64, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 64; ++j) s[64 + j] = __uint_as_float(r[j]);
            }
            // ---- mask (edge tiles only), row maximum; the row's base moves if it outgrew it ----
            const int j0 = (kb_lo + i) * kKT;
            if (!(row_ok && j0 >= lo_row && j0 + kKT - 1 <= pos_row)) {
#pragma unroll
                for (int j = 0; j < kKT; ++j) {
                    const int key = j0 + j;
                    const bool valid = row_ok && key >= lo_row && key <= pos_row;
                    s[j] = valid ? s[j] : -INFINITY;
                }
            }
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // short chains
#pragma unroll
            for (int j = 0; j < kKT; j += 8) {
                mx4[0] = max3(mx4[0], s[j], s[j + 1]);
                mx4[1] = max3(mx4[1], s[j + 2], s[j + 3]);
                mx4[2] = max3(mx4[2], s[j + 4], s[j + 5]);
                mx4[3] = max3(mx4[3], s[j + 6], s[j + 7]);
            }
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * p.scale_log2;
            const bool move = mx > m_base + kLazy;
            float f = 1.f;  // factor of the row's earlier output and sum
            if (move) {
                f = exp2f(m_base - mx);  // 0 while the row had no key (m_base = -inf)
                m_base = mx;
                l_run *= f;
            }
            const float mu = (m_base == -INFINITY) ? 0.f : m_base;
            __syncwarp();  // the row-dependent branches above rejoin before the TMEM stores
            // ---- P row: exponentials two lanes per instruction, into TMEM over S's columns ----
            {
                const uint64_t sc2 = f2(p.scale_log2, p.scale_log2), nmu2 = f2(-mu, -mu);
                uint64_t acc[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
                for (int c = 0; c < kKT / 32; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const uint64_t x = f2_fma(f2(s[c * 32 + 2 * u], s[c * 32 + 2 * u + 1]), sc2, nmu2);
                        uint64_t e;
                        if ((u & 3) == 3) {
                            e = exp2_fma_x2(x);
                        } else {
                            float a0, a1;
                            f2_split(x, a0, a1);
                            e = f2(ex2_approx(a0), ex2_approx(a1));
                        }
                        acc[u & 1] = f2_add(acc[u & 1], e);
                        float e0, e1;
                        f2_split(e, e0, e1);
                        pk[u] = pack_bf16x2(e0, e1);
                    }
                    tmem_st16(s_col + 16 * c, pk);
                }
                float a0, a1, b0, b1;
                f2_split(acc[0], a0, a1);
                f2_split(acc[1], b0, b1);
                l_run += (a0 + a1) + (b0 + b1);
            }
            // ---- the row's earlier output to the new base (the product into it is done) -------
            if (__any_sync(0xffffffffu, move) && i > 0) {
#pragma unroll
                for (int c = 0; c < kD / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(o_col + 32 * c, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * f);
                    tmem_st32(o_col + 32 * c, r);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_PFULL + qt));
        }
        if (ok) ok = wait_or_abort(bar(B_ODONE + qt), 0, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            uint4 *dst = reinterpret_cast<uint4 *>(p.o + (((size_t)b * p.T + t_row) * p.Hq + h_row) * kD);
#pragma unroll
            for (int c = 0; c < kD / 32; ++c) {
                __syncwarp();  // converged for the TMEM load after the row-dependent stores
                uint32_t r[32];
                tmem_ld32(o_col + 32 * c, r);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float *v = reinterpret_cast<const float *>(r + 8 * q4);
                        dst[c * 4 + q4] = make_uint4(pack_bf16x2(v[0] * inv, v[1] * inv),
                                                     pack_bf16x2(v[2] * inv, v[3] * inv),
                                                     pack_bf16x2(v[4] * inv, v[5] * inv),
                                                     pack_bf16x2(v[6] * inv, v[7] * inv));
                    }
                }
            }
        } else if (lane == 0) {
            atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// The SWA ring write of a prompt that followed a cached prefix, after the attention kernel has
// read every prefix key: the last R*64 positions of the prompt (the ones the ring keeps), one
// 16-byte chunk of K or V per thread.
template <int D>
__global__ void __launch_bounds__(256) attn_prefill_ring_write_kernel(const TcParams p) {
    constexpr int kD = D;
    griddep_launch_dependents();
    griddep_wait();  // the attention kernel has read the ring
    const int ring = p.ring_pages * kPT;
    const int t_lo = p.T > ring ? p.T - ring : 0;
    constexpr int CH = kD / 8;
    const long long n = (long long)p.B * (p.T - t_lo) * p.Hkv * 2 * CH;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
         idx += (long long)gridDim.x * blockDim.x) {
        const int chk = (int)(idx % CH);
        long long r = idx / CH;
        const bool is_v = (r & 1) != 0;
        r >>= 1;
        const int g = (int)(r % p.Hkv);
        r /= p.Hkv;
        const int t = t_lo + (int)(r % (p.T - t_lo));
        const int b = (int)(r / (p.T - t_lo));
        int L0 = p.prefix_lens ? p.prefix_lens[b] : 0;
        if (L0 < 0 || (L0 % kPT) != 0) L0 = 0;  // reported by the attention kernel
        const int li = (L0 + t) % ring;
        const int lp = li / kPT;
        const int pg = lp < p.max_pages ? p.page_table[(size_t)b * p.max_pages + lp] : -1;
        if (pg < 0 || pg >= p.n_pages) {
            atomicOr(&g_err, HMD_DEVERR_PAGE);
            continue;
        }
        const size_t srco = (((size_t)b * p.T + t) * p.Hkv + g) * kD + chk * 8;
        const size_t dsto = (((size_t)pg * p.Hkv + g) * kPT + (li % kPT)) * kD + chk * 8;
        *reinterpret_cast<uint4 *>((is_v ? p.v_pool : p.k_pool) + dsto) =
            *reinterpret_cast<const uint4 *>((is_v ? p.v : p.k) + srco);
    }
}

}  // namespace

bool attn_prefill_tc_supported(int d, int page_tokens, int group) {
    const bool g_ok = group == 1 || group == 2 || group == 4 || group == 8 || group == 16;
    return (d == 64 || d == 128) && page_tokens == kPT && g_ok;
}

namespace {
template <int D>
cudaError_t launch_tc(const AttnPrefillArgs &a, cudaStream_t s) {
    constexpr uint32_t kSmem = Smem<D>::BYTES;
    const cudaError_t attr_err = once_per_device([] {
        cudaError_t e = cudaFuncSetAttribute(attn_prefill_tc_kernel<D, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)Smem<D>::BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(attn_prefill_tc_kernel<D, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Smem<D>::BYTES);
        return e;
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap tmk, tmv, tmpk, tmpv;
    const long long n_tok = (long long)a.B * a.T;
    if (!make_tmap_tokens_sw128(&tmk, const_cast<void *>(a.k), n_tok, a.Hkv, D) ||
        !make_tmap_tokens_sw128(&tmv, const_cast<void *>(a.v), n_tok, a.Hkv, D))
        return cudaErrorInvalidValue;
    if (a.prefix_lens) {
        if (!make_tmap_pool_sw128(&tmpk, a.k_pool, a.n_pages, a.Hkv, D) ||
            !make_tmap_pool_sw128(&tmpv, a.v_pool, a.n_pages, a.Hkv, D))
            return cudaErrorInvalidValue;
    } else {
        tmpk = tmk;  // not read
        tmpv = tmv;
    }
    TcParams p;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.k = static_cast<const __nv_bfloat16 *>(a.k);
    p.v = static_cast<const __nv_bfloat16 *>(a.v);
    p.k_pool = static_cast<__nv_bfloat16 *>(a.k_pool);
    p.v_pool = static_cast<__nv_bfloat16 *>(a.v_pool);
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.page_table = a.page_table;
    p.prefix_lens = a.prefix_lens;
    // with a prefix, SWA prompt tokens would overwrite ring slots of prefix keys that other
    // CTAs still read: their cache write moves to a kernel that runs after the attention
    p.defer_write = (a.swa && a.prefix_lens) ? 1 : 0;
    p.B = a.B; p.T = a.T; p.Hq = a.Hq; p.Hkv = a.Hkv;
    p.G = a.Hq / a.Hkv;
    p.QT = kRows / p.G;
    p.n_qb = (a.T + 2 * p.QT - 1) / (2 * p.QT);
    p.window = a.window; p.swa = a.swa ? 1 : 0;
    p.ring_pages = a.swa ? (a.window + kPT - 1) / kPT : 0;
    p.max_pages = a.max_pages; p.n_pages = a.n_pages;
    p.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    const long long grid = (long long)p.n_qb * a.B * a.Hkv;
    cudaError_t e = a.prefix_lens
        ? launch_pdl(attn_prefill_tc_kernel<D, true>, dim3((unsigned)grid), dim3(kThreads), kSmem,
                     s, tmk, tmv, tmpk, tmpv, p)
        : launch_pdl(attn_prefill_tc_kernel<D, false>, dim3((unsigned)grid), dim3(kThreads), kSmem,
                     s, tmk, tmv, tmpk, tmpv, p);
    if (e != cudaSuccess || !p.defer_write) return e;
    const int ring = p.ring_pages * kPT;
    const long long n = (long long)a.B * std::min(a.T, ring) * a.Hkv * 2 * (D / 8);
    const unsigned blocks = (unsigned)std::min<long long>((n + 255) / 256, 148LL * 16);
    return launch_pdl(attn_prefill_ring_write_kernel<D>, dim3(blocks), dim3(256), 0, s, p);
}
}  // namespace

cudaError_t launch_attn_prefill_tc(const AttnPrefillArgs &a, cudaStream_t s) {
    if (a.B == 0 || a.T == 0) return cudaSuccess;
    if (a.d == 128) return launch_tc<128>(a, s);
    if (a.d == 64) return launch_tc<64>(a, s);
    return cudaErrorInvalidValue;
}

bool attn_prefill_supported(int d, int page_tokens, int group) {
    return attn_prefill_tc_supported(d, page_tokens, group);
}

cudaError_t launch_attn_prefill(const AttnPrefillArgs &a, cudaStream_t s) {
    return launch_attn_prefill_tc(a, s);
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

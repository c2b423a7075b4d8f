// Delta-rule decode step (GDN and KDA), one token per sequence.
//
// The pages name GDN (scalar gate) and KDA (channel-wise gate) as the two O(n) recurrent mixers
// of every supernet layer ("Super Apriel: One Checkpoint, Many Speeds", abstract; gist.science
// technical summary, section 2a). With the state stored as M[d_k][d_v] (M = S^T for GDN, M = S
// for KDA), one token of either standard definition is
//     M' = Diag(a) M,   u = beta (v - M'^T k),   M = M' + k u^T,   o = scale * M^T q,
// a = exp(log_gate) (a scalar broadcast over d_k for GDN). Since M^T q = M'^T q + u (k.q), one
// read of M gives both column reductions M'^T k and M'^T q, and one write stores the update:
// the state crosses HBM exactly twice (read + write), which is the algorithmic minimum.
//
// Work split: one CTA of 128 threads per (sequence, head, 32-column slice of d_v). The slice
// ([d_k][32] fp32, 16 KiB at d_k = 128) arrives by one 2-D TMA box into shared memory and leaves
// by one TMA store after the update (in place, or to another slot: a speculative draft step
// writes a fresh slot so that rejecting it is a choice of slot, not a copy), so each CTA holds few registers and many CTAs per
// SM keep their slices in flight. A thread owns 4 adjacent columns (one 16-byte vector) of
// d_k/16 rows; column sums are reduced over rows with warp shuffles (xor 8, 16), then across the
// 4 warps through shared memory. No tensor cores: the step is ~1 flop per byte, far below any
// ridge.
#include <cuda.h>

#include "kernels.h"
#include "ptx.cuh"
#include "../../include/hmd.h"

namespace hmd {
namespace {

__device__ unsigned int g_err;

constexpr int kThreads = 128;
constexpr int kColThreads = 8;                     // float4 columns across a slice
constexpr int kSliceCols = 4 * kColThreads;        // 32 columns of d_v per CTA
constexpr int kRowThreads = kThreads / kColThreads;  // 16 row groups
constexpr int kWarps = kThreads / 32;

template <bool BF16>
__device__ __forceinline__ float act(const void *p, size_t i) {
    if constexpr (BF16) {
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    } else {
        return reinterpret_cast<const float *>(p)[i];
    }
}

// CHAIN: nq tokens per launch along a slot chain (a.nq, a.chain); otherwise one token with
// a.nq == 1, compiled without the token loop.
template <int DK, bool BF16, bool CHAIN>
__global__ void __launch_bounds__(kThreads) delta_decode_kernel(const __grid_constant__ CUtensorMap tm,
                                                                const DeltaDecodeArgs a,
                                                                int n_slices) {
    const int nq = CHAIN ? a.nq : 1;
    constexpr int RPT = DK / kRowThreads;  // rows per thread
    __shared__ __align__(128) float S[DK][kSliceCols];
    __shared__ float sk[DK], sq[DK], sa[DK];
    __shared__ float red[kWarps][kColThreads][9];
    __shared__ float nrm[kWarps][2];
    __shared__ __align__(8) uint64_t bar;
    __shared__ int s_ok;
    const int slice = blockIdx.x % n_slices;
    const int bh = blockIdx.x / n_slices;
    const int ri = bh / a.H;  // row of the launch: sequence ri, or rows[ri] for a sub-batch
    const int h = bh - ri * a.H;
    const int tid = threadIdx.x;
    const int ct = tid % kColThreads;
    const int rt = tid / kColThreads;
    const int col = slice * kSliceCols + ct * 4;
    const bool active = col < a.dv;

    if (tid == 0) prefetch_tmap(&tm);
    griddep_launch_dependents();
    griddep_wait();  // q, k, v, gates and the state may come from the previous kernel
    const int b = a.rows ? a.rows[ri] : ri;
    // the slot read before token 0, and the slot written after token t
    const int src = CHAIN ? a.chain[b] : (a.slots ? a.slots[b] : b);
    auto dst_of = [&](int t) {
        return CHAIN ? a.chain[(size_t)(t + 1) * a.B + b] : (a.dst_slots ? a.dst_slots[b] : src);
    };
    if (tid == 0) {
        const int slot = src;
        bool ok = slot >= 0 && slot < a.n_slots;
        for (int t = 0; t < nq; ++t) {
            const int dst = dst_of(t);
            ok = ok && dst >= 0 && dst < a.n_slots;
        }
        s_ok = ok;
        if (ok) {
            const uint32_t bb = smem_u32(&bar);
            mbar_init(bb, 1);
            fence_barrier_init();
            mbar_arrive_expect_tx(bb, DK * kSliceCols * 4);
            if ((int)blockIdx.x != a.skip.cta)  // a test may arm this barrier with no copy
                tma_load_2d(smem_u32(&S[0][0]), &tm, bb, slice * kSliceCols, (slot * a.H + h) * DK);
        } else {
            atomicOr(&g_err, HMD_DEVERR_SLOT);
        }
    }
    const bool fused = a.act.A_log != nullptr;  // raw projections: activate them here
    for (int t = 0; t < nq; ++t) {  // body not re-indented: one token per iteration
    const size_t tok = ((size_t)b * nq + t) * a.H + h;
    const float rate = fused ? expf(a.act.A_log[h]) : 0.f;
    if (a.kind == HMD_GDN) {
        float lg = a.log_gate[tok];
        if (fused) lg = -rate * hmd_softplus(lg + a.act.dt_bias[h]);
        const float g = expf(lg);
        for (int i = tid; i < DK; i += kThreads) sa[i] = g;
    } else {
        for (int i = tid; i < DK; i += kThreads) {
            float lg = a.log_gate[tok * DK + i];
            if (fused) lg = -rate * hmd_softplus(lg + a.act.dt_bias[(size_t)h * DK + i]);
            sa[i] = expf(lg);
        }
    }
    float ssk = 0.f, ssq = 0.f;
    for (int i = tid; i < DK; i += kThreads) {
        const float kv = act<BF16>(a.k, tok * DK + i), qv = act<BF16>(a.q, tok * DK + i);
        sk[i] = kv;
        sq[i] = qv;
        ssk += kv * kv;
        ssq += qv * qv;
    }
    float vv[4] = {0.f, 0.f, 0.f, 0.f};
    if (active) {
#pragma unroll
        for (int c = 0; c < 4; ++c) vv[c] = act<BF16>(a.v, tok * a.dv + col + c);
    }
    float beta = a.beta[tok];
    if (fused) {
        beta = 1.f / (1.f + expf(-beta));
        // L2 norms of k and q over d_k: warp sums, then the kWarps partials
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
            ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
        }
        if ((tid & 31) == 0) {
            nrm[tid >> 5][0] = ssk;
            nrm[tid >> 5][1] = ssq;
        }
        __syncthreads();
        float tk = 0.f, tq = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            tk += nrm[w][0];
            tq += nrm[w][1];
        }
        const float fk = rsqrtf(tk + a.act.eps), fq = rsqrtf(tq + a.act.eps);
        for (int i = tid; i < DK; i += kThreads) {
            sk[i] *= fk;
            sq[i] *= fq;
        }
    }
    __syncthreads();
    if (!s_ok) return;
    // the CTA gives up together: one thread's timeout decides for all of them
    if (t == 0 && __syncthreads_or(!mbar_wait_bounded(smem_u32(&bar), 0, a.skip.wait_ns))) {
        if (tid == 0) {
            atomicOr(&g_err, HMD_DEVERR_TIMEOUT);
            // the copy may still land: let it finish (bounded) before the shared memory goes
            (void)mbar_wait_bounded(smem_u32(&bar), 0, a.skip.wait_ns);
        }
        return;  // nothing was written; the state slice is left as it was
    }

    // M' = Diag(a) M and the partial column sums of M'^T k, M'^T q, k.q.
    float w[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f}, kq = 0.f;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rt + r * kRowThreads;
        const float ai = sa[i], ki = sk[i], qi = sq[i];
        float4 m = *reinterpret_cast<const float4 *>(&S[i][ct * 4]);
        m.x *= ai; m.y *= ai; m.z *= ai; m.w *= ai;
        w[0] += ki * m.x; w[1] += ki * m.y; w[2] += ki * m.z; w[3] += ki * m.w;
        pq[0] += qi * m.x; pq[1] += qi * m.y; pq[2] += qi * m.z; pq[3] += qi * m.w;
        kq += ki * qi;
    }
#pragma unroll
    for (int off = 8; off < 32; off <<= 1) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            w[c] += __shfl_xor_sync(0xffffffffu, w[c], off);
            pq[c] += __shfl_xor_sync(0xffffffffu, pq[c], off);
        }
        kq += __shfl_xor_sync(0xffffffffu, kq, off);
    }
    const int warp = tid >> 5, lane = tid & 31;
    if (lane < kColThreads) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            red[warp][lane][c] = w[c];
            red[warp][lane][4 + c] = pq[c];
        }
        red[warp][lane][8] = kq;
    }
    if (t > 0 && tid == 0) bulk_wait_group_read0();  // token t-1's store has read S
    __syncthreads();
    float W[4] = {0.f, 0.f, 0.f, 0.f}, PQ[4] = {0.f, 0.f, 0.f, 0.f}, KQ = 0.f;
#pragma unroll
    for (int wi = 0; wi < kWarps; ++wi) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            W[c] += red[wi][ct][c];
            PQ[c] += red[wi][ct][4 + c];
        }
        KQ += red[wi][ct][8];
    }
    float u[4], o[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        u[c] = beta * (vv[c] - W[c]);
        o[c] = a.scale * (PQ[c] + u[c] * KQ);
    }
    // M = M' + k u^T, in place
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int i = rt + r * kRowThreads;
        const float ai = sa[i], ki = sk[i];
        float4 m = *reinterpret_cast<const float4 *>(&S[i][ct * 4]);
        m.x = ai * m.x + ki * u[0];
        m.y = ai * m.y + ki * u[1];
        m.z = ai * m.z + ki * u[2];
        m.w = ai * m.w + ki * u[3];
        *reinterpret_cast<float4 *>(&S[i][ct * 4]) = m;
    }
    if (rt == 0 && active) {
        if constexpr (BF16) {
            uint2 pk;
            pk.x = pack_bf16x2(o[0], o[1]);
            pk.y = pack_bf16x2(o[2], o[3]);
            *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(a.o) + tok * a.dv + col) = pk;
        } else {
            *reinterpret_cast<float4 *>(reinterpret_cast<float *>(a.o) + tok * a.dv + col) =
                make_float4(o[0], o[1], o[2], o[3]);
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        tma_store_2d(&tm, smem_u32(&S[0][0]), slice * kSliceCols, (dst_of(t) * a.H + h) * DK);
        bulk_commit_group();
    }
    }  // tokens
    if (tid == 0) bulk_wait_group_read0();  // shared memory must outlive the last store's read
}

template <int DK>
cudaError_t launch_dk(const DeltaDecodeArgs &a, cudaStream_t s) {
    const int n_slices = (a.dv + kSliceCols - 1) / kSliceCols;
    const long long grid = (long long)(a.rows ? a.n_rows : a.B) * a.H * n_slices;
    if (grid <= 0) return cudaSuccess;
    // the state cache as a 2-D tensor [n_slots*H*DK rows][dv] fp32, read in 32-column boxes
    CUtensorMap tm;
    if (!make_tmap_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.state, a.dv,
                      (long long)a.n_slots * a.H * DK, kSliceCols, DK))
        return cudaErrorInvalidValue;
    const bool chain = a.chain != nullptr;
    if (a.bf16)
        return chain ? launch_pdl(delta_decode_kernel<DK, true, true>, dim3((unsigned)grid),
                                  dim3(kThreads), 0, s, tm, a, n_slices)
                     : launch_pdl(delta_decode_kernel<DK, true, false>, dim3((unsigned)grid),
                                  dim3(kThreads), 0, s, tm, a, n_slices);
    return chain ? launch_pdl(delta_decode_kernel<DK, false, true>, dim3((unsigned)grid),
                              dim3(kThreads), 0, s, tm, a, n_slices)
                 : launch_pdl(delta_decode_kernel<DK, false, false>, dim3((unsigned)grid),
                              dim3(kThreads), 0, s, tm, a, n_slices);
}

}  // namespace

bool delta_decode_supported(int dk, int dv) {
    const bool dk_ok = dk == 16 || dk == 32 || dk == 64 || dk == 128 || dk == 256;
    return dk_ok && dv >= 4 && dv <= 1024 && dv % 4 == 0;
}

cudaError_t launch_delta_decode(const DeltaDecodeArgs &a, cudaStream_t s) {
    switch (a.dk) {
        case 16: return launch_dk<16>(a, s);
        case 32: return launch_dk<32>(a, s);
        case 64: return launch_dk<64>(a, s);
        case 128: return launch_dk<128>(a, s);
        case 256: return launch_dk<256>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

uint32_t delta_decode_read_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_err, sizeof v) != cudaSuccess) return 0;
    if (clear && v) {
        const unsigned int z = 0;
        cudaMemcpyToSymbol(g_err, &z, sizeof z);
    }
    return v;
}

}  // namespace hmd

// Chunked (WY / UT-transform) prefill of the delta-rule mixers (GDN, KDA).
//
// The pages name the two recurrent mixers and their O(n) cost ("Super Apriel: One Checkpoint,
// Many Speeds", abstract; gist.science technical summary, section 2a); the recurrence is the
// standard one (see delta_decode.cu). Over a chunk of C tokens starting from state M0, with
// per-channel cumulative log-gates G[r][i] = sum_{s<=r} log a_{s,i}, it is exactly
//   A[r][s] = beta_r sum_i k_ri k_si e^(G_ri - G_si)  (s < r)
//   T = (I + A)^{-1} Diag(beta)                    (unit lower-triangular solve)
//   U = T (V - Kt M0),  Kt = k * exp(G)            (U[r] is token r's delta-rule write)
//   P[r][s] = sum_i q_ri k_si e^(G_ri - G_si)  (s <= r),  O = Qt M0 + P U,  Qt = q * exp(G)
//   M_C = Diag(exp(G_C)) M0 + sum_s (k_s exp(G_C - G_s))^T U_s,  G_C = G of the chunk's last token.
// The decays e^(G_r - G_s) are formed as e^G_r e^-G_s while every |G| of the chunk is at most
// kPrefillFactorRange (both factors then stay inside fp32's range) and directly otherwise, so
// any gate is accepted.
//
// bf16 inputs with d_k = d_v = 128 and C = 64 run on the tensor cores in two passes
// (delta_prefill_tc.cu).
// This file holds the generic path: one CTA per (sequence, head, 32-column slice of d_v) runs
// the chunks in order with the slice of the state resident in shared memory, all arithmetic in
// fp32 on CUDA cores (so fp32 inputs keep fp32 accuracy). The k-side products (A, T, P) do
// not depend on d_v and are recomputed by every slice's CTA.
#include "kernels.h"
#include "ptx.cuh"
#include "../../include/hmd.h"

namespace hmd {
namespace {

__device__ unsigned int g_err;

constexpr int kC = 64;          // chunk length
constexpr int kThreads = 256;
constexpr int kSlice = 32;      // d_v columns per CTA

template <bool BF16>
__device__ __forceinline__ float ld_act(const void *p, size_t i) {
    if constexpr (BF16) {
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    } else {
        return reinterpret_cast<const float *>(p)[i];
    }
}

size_t generic_smem_bytes(int dk, int dvs) {
    return sizeof(float) * ((size_t)4 * kC * dk + 2 * (size_t)kC * dvs + (size_t)dk * dvs +
                            3 * (size_t)kC * kC + 2 * (size_t)dk + kC);
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads) prefill_generic_kernel(const DeltaPrefillArgs a,
                                                                   int n_slices, int dvs) {
    extern __shared__ float sm[];
    const int dk = a.dk, dv = a.dv;
    float *Kr = sm;                         // [C][dk] k
    float *Qr = Kr + kC * dk;               // [C][dk] q
    float *Eg = Qr + kC * dk;               // [C][dk] e^G
    float *Gx = Eg + kC * dk;               // [C][dk] e^-G (factored chunks) or G (direct ones)
    float *Vs = Gx + kC * dk;               // [C][dvs]
    float *Us = Vs + kC * dvs;              // [C][dvs]
    float *Ms = Us + kC * dvs;              // [dk][dvs]
    float *Am = Ms + dk * dvs;              // [C][C]
    float *Tm = Am + kC * kC;               // [C][C]
    float *Pm = Tm + kC * kC;               // [C][C]
    float *egl = Pm + kC * kC;              // [dk] e^G_C
    float *gl = egl + dk;                   // [dk] G_C
    float *bt = gl + dk;                    // [C] beta

    const int slice = blockIdx.x % n_slices;
    const int bh = blockIdx.x / n_slices;
    const int b = bh / a.H, h = bh - b * a.H;
    const int j0 = slice * dvs;
    const int ncols = min(dvs, dv - j0);
    const int tid = threadIdx.x;
    const int slot = a.slots ? a.slots[b] : b;
    if (slot < 0 || slot >= a.n_slots) {
        if (tid == 0) atomicOr(&g_err, HMD_DEVERR_SLOT);
        return;
    }
    float *Mg = a.state + ((size_t)slot * a.H + h) * (size_t)dk * dv;
    for (int idx = tid; idx < dk * dvs; idx += kThreads) {
        const int i = idx / dvs, jj = idx % dvs;
        Ms[idx] = jj < ncols ? Mg[(size_t)i * dv + j0 + jj] : 0.f;
    }

    for (int t0 = 0; t0 < a.T; t0 += kC) {
        const int n = min(kC, a.T - t0);
        __syncthreads();  // previous chunk fully consumed
        // gates: G per channel, and whether the factored form stays inside fp32's range
        bool out_of_range = false;
        for (int i = tid; i < dk; i += kThreads) {
            float g = 0.f;
            for (int r = 0; r < kC; ++r) {
                if (r < n) {
                    const size_t tok = ((size_t)b * a.T + t0 + r) * a.H + h;
                    g += a.kind == HMD_GDN ? a.log_gate[tok] : a.log_gate[tok * dk + i];
                }
                Gx[r * dk + i] = g;
                out_of_range |= g < -kPrefillFactorRange || g > kPrefillFactorRange;
            }
            gl[i] = g;
            egl[i] = expf(g);
        }
        const bool direct = __syncthreads_or(out_of_range);
        // q, k, e^G and (factored chunks) e^-G, the v slice, beta
        for (int idx = tid; idx < kC * dk; idx += kThreads) {
            const int r = idx / dk, i = idx % dk;
            const size_t tok = ((size_t)b * a.T + t0 + r) * a.H + h;
            const float g = Gx[idx];
            Kr[idx] = r < n ? ld_act<BF16>(a.k, tok * dk + i) : 0.f;
            Qr[idx] = r < n ? ld_act<BF16>(a.q, tok * dk + i) : 0.f;
            Eg[idx] = expf(g);
            if (!direct) Gx[idx] = expf(-g);
        }
        for (int idx = tid; idx < kC * dvs; idx += kThreads) {
            const int r = idx / dvs, jj = idx % dvs;
            const size_t tok = ((size_t)b * a.T + t0 + r) * a.H + h;
            Vs[idx] = (r < n && jj < ncols) ? ld_act<BF16>(a.v, tok * dv + j0 + jj) : 0.f;
        }
        for (int r = tid; r < kC; r += kThreads)
            bt[r] = r < n ? a.beta[((size_t)b * a.T + t0 + r) * a.H + h] : 0.f;
        __syncthreads();
        // A (strictly lower, beta-scaled) and P (lower incl. diagonal):
        // sum_i x_ri k_si e^(G_ri - G_si) with x = k (A) or q (P), the decay as e^G_r e^-G_s in a
        // factored chunk, else formed directly
        for (int idx = tid; idx < kC * kC; idx += kThreads) {
            const int r = idx / kC, s = idx % kC;
            float av = 0.f, pv = 0.f;
            if (s <= r && r < n) {
                for (int i = 0; i < dk; ++i) {
                    const float d = direct ? expf(Gx[r * dk + i] - Gx[s * dk + i])
                                           : Eg[r * dk + i] * Gx[s * dk + i];
                    const float ks = Kr[s * dk + i] * d;
                    av += Kr[r * dk + i] * ks;
                    pv += Qr[r * dk + i] * ks;
                }
            }
            Am[idx] = s < r ? bt[r] * av : 0.f;
            Pm[idx] = pv;
        }
        __syncthreads();
        // T = (I + A)^{-1} Diag(beta), one column per thread by forward substitution
        for (int c = tid; c < kC; c += kThreads) {
            for (int r = 0; r < kC; ++r) {
                float x = 0.f;
                if (r >= c && r < n) {
                    x = r == c ? bt[r] : 0.f;
                    for (int s = c; s < r; ++s) x -= Am[r * kC + s] * Tm[s * kC + c];
                }
                Tm[r * kC + c] = x;
            }
        }
        __syncthreads();
        // Z = V - Kt M0 (Kt = k e^G), into Us
        for (int idx = tid; idx < kC * dvs; idx += kThreads) {
            const int r = idx / dvs, jj = idx % dvs;
            float acc = Vs[idx];
            for (int i = 0; i < dk; ++i) acc -= Kr[r * dk + i] * Eg[r * dk + i] * Ms[i * dvs + jj];
            Us[idx] = acc;
        }
        __syncthreads();
        // U = T Z (= T V - W M0 with W = T Kt), into Vs
        for (int idx = tid; idx < kC * dvs; idx += kThreads) {
            const int r = idx / dvs, jj = idx % dvs;
            float acc = 0.f;
            for (int s = 0; s <= r; ++s) acc += Tm[r * kC + s] * Us[s * dvs + jj];
            Vs[idx] = acc;
        }
        __syncthreads();
        // O = Qt M0 + P U (Qt = q e^G)
        for (int idx = tid; idx < kC * dvs; idx += kThreads) {
            const int r = idx / dvs, jj = idx % dvs;
            if (r >= n || jj >= ncols) continue;
            float acc = 0.f;
            for (int i = 0; i < dk; ++i) acc += Qr[r * dk + i] * Eg[r * dk + i] * Ms[i * dvs + jj];
            for (int s = 0; s <= r; ++s) acc += Pm[r * kC + s] * Vs[s * dvs + jj];
            acc *= a.scale;
            const size_t oi = (((size_t)b * a.T + t0 + r) * a.H + h) * dv + j0 + jj;
            if constexpr (BF16) {
                reinterpret_cast<__nv_bfloat16 *>(a.o)[oi] = __float2bfloat16_rn(acc);
            } else {
                reinterpret_cast<float *>(a.o)[oi] = acc;
            }
        }
        __syncthreads();
        // M_C = Diag(e^G_C) M0 + sum_s (k_s e^(G_C - G_s))^T U_s
        for (int idx = tid; idx < dk * dvs; idx += kThreads) {
            const int i = idx / dvs, jj = idx % dvs;
            float acc = 0.f;
            for (int s = 0; s < n; ++s) {
                const float d = direct ? expf(gl[i] - Gx[s * dk + i]) : egl[i] * Gx[s * dk + i];
                acc += Kr[s * dk + i] * d * Vs[s * dvs + jj];
            }
            Ms[idx] = egl[i] * Ms[idx] + acc;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < dk * dvs; idx += kThreads) {
        const int i = idx / dvs, jj = idx % dvs;
        if (jj < ncols) Mg[(size_t)i * dv + j0 + jj] = Ms[idx];
    }
}

}  // namespace

bool delta_prefill_supported(int dk, int dv, bool bf16, int chunk) {
    (void)bf16;
    const bool dk_ok = dk % 16 == 0 && dk >= 16 && dk <= 128;
    const bool dv_ok = dv % 16 == 0 && dv >= 16 && dv <= 128;
    return dk_ok && dv_ok && chunk == kC;
}

cudaError_t launch_delta_prefill(const DeltaPrefillArgs &a, cudaStream_t s) {
    const int dvs = a.dv < kSlice ? a.dv : kSlice;
    const int n_slices = (a.dv + dvs - 1) / dvs;
    const size_t smem = generic_smem_bytes(a.dk, dvs);
    const long long grid = (long long)a.B * a.H * n_slices;
    if (grid <= 0) return cudaSuccess;
    cudaError_t e;
    if (a.bf16) {
        e = cudaFuncSetAttribute(prefill_generic_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        prefill_generic_kernel<true><<<(unsigned)grid, kThreads, smem, s>>>(a, n_slices, dvs);
    } else {
        e = cudaFuncSetAttribute(prefill_generic_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        prefill_generic_kernel<false><<<(unsigned)grid, kThreads, smem, s>>>(a, n_slices, dvs);
    }
    return cudaGetLastError();
}

uint32_t delta_prefill_read_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_err, sizeof v) != cudaSuccess) return 0;
    if (clear && v) {
        const unsigned int z = 0;
        cudaMemcpyToSymbol(g_err, &z, sizeof z);
    }
    return v;
}

}  // namespace hmd

// Internal launchers shared between the C-ABI layer (hmd_api.cu) and the kernel files.
// Every launcher validates nothing (the API layer already did) and returns the launch status.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "../../include/hmd.h"

namespace hmd {

// The chunked prefill factors each decay e^{G_r - G_s} into e^{G_r} and e^{-G_s} (so that the
// chunk's products are plain matrix products) while every cumulative in-chunk log-gate |G| is at
// most this bound: both factors then stay inside fp32's normal range (e^88 overflows). Chunks
// beyond it form the decays directly.
constexpr float kPrefillFactorRange = 80.f;

// Runs f() for the current device until it succeeds once, then returns that result on every
// later call there. Kernel attributes (the dynamic shared-memory limit) and device properties
// belong to one device, so a process that drives several GPUs sets and reads them per device.
// A CUDA error (for instance a transient failure to set an attribute) is returned to its caller
// and not kept: f() runs again on the next call. When the current device cannot be determined,
// f() runs uncached.
constexpr int kMaxDevices = 64;
template <typename R>
inline bool once_cacheable(const R &) { return true; }
inline bool once_cacheable(const cudaError_t &e) { return e == cudaSuccess; }
template <typename F>
auto once_per_device(F f) -> decltype(f()) {
    using R = decltype(f());
    static std::mutex mu;
    static std::atomic<bool> done[kMaxDevices];
    static R results[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return f();
    }
    if (done[dev].load(std::memory_order_acquire)) return results[dev];
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev].load(std::memory_order_relaxed)) {
        const R r = f();
        if (!once_cacheable(r)) return r;
        results[dev] = r;
        done[dev].store(true, std::memory_order_release);
    }
    return results[dev];
}

// Records `s` as this host thread's last error (read by hmd_last_error) and returns it; for
// entry points defined outside the API file.
hmd_status_t record_status(hmd_status_t s);

// One-shot fault injection for the failure-detection tests (hmd_test_arm_copy_skip): the next
// launch of `kernel` on this host thread has CTA `cta` arm its first copy barrier without
// issuing the copy, and every bounded wait in it gives up after wait_ns.
struct CopySkip {
    int cta = -1;                              // -1: nothing armed
    unsigned long long wait_ns = 2000000000ull;  // the normal 2 s limit
};
CopySkip take_copy_skip(int kernel);

// Launches `kernel` on stream s with programmatic stream serialisation: it may be scheduled
// while the previous kernel in the stream drains, and waits for it (griddep_wait) before its
// first global-memory access, so results are those of an ordinary launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// TMA tensor map over a 2-D row-major tensor, boxes of [box_rows][box_cols], no swizzle.
bool make_tmap_2d(CUtensorMap *m, CUtensorMapDataType dt, int esize, void *base, long long cols,
                  long long rows, int box_cols, int box_rows);

// [n_tok][heads][d] bf16 as (d, heads, n_tok) in 64 x 1 x 64 boxes, 128-byte swizzle.
bool make_tmap_tokens_sw128(CUtensorMap *m, void *base, long long n_tok, int heads, int d);
bool make_tmap_bthd(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, int B,
                    int T, int H, int d, int box_d, bool sw128);
bool make_tmap_pool_sw128(CUtensorMap *m, void *pool, int n_pages, int heads, int d);

// Input activations of the delta-rule mixers, fused into their kernels when A_log is set: the
// kernel then reads raw q, k (L2-normalised over d_k with eps), beta logits (sigmoid) and gate
// logits (log-gate = -exp(A_log[h]) * softplus(logit + dt_bias), dt_bias [H] for GDN, [H][dk]
// for KDA). A_log == nullptr: the inputs are already q, k, beta and log-gates.
struct DeltaAct {
    const float *A_log = nullptr;
    const float *dt_bias = nullptr;
    float eps = 0.f;
};

// softplus(x) = log(1 + e^x) = max(x, 0) + log(1 + y), y = e^-|x| in (0, 1]; log(1 + y) is the
// series y - y^2/2 + y^3/3 - y^4/4 while y < 1/64 (next term y^5/5, a relative 3e-8), else
// log(1 + y), where 1 + y keeps y to a relative 4e-6. Both are computed and one is selected,
// so a warp never diverges on it.
__device__ __forceinline__ float hmd_softplus(float x) {
    const float y = __expf(-fabsf(x));
    const float ser = y * (1.f - y * (0.5f - y * (1.f / 3.f - 0.25f * y)));
    const float lg = __logf(1.f + y);
    return fmaxf(x, 0.f) + (y < 0.015625f ? ser : lg);
}

struct DeltaDecodeArgs {
    int kind;  // 2 = KDA (per-channel gate), 3 = GDN (scalar gate)
    int B, H, dk, dv;
    bool bf16;  // activations bf16 (else fp32)
    const void *q, *k, *v;
    const float *beta, *log_gate;
    float *state;
    int n_slots;
    const int32_t *slots;
    const int32_t *dst_slots;  // where the updated state goes (NULL: back to slots, in place)
    void *o;
    float scale;
    const int32_t *rows = nullptr;  // batch rows to run (device, n_rows of them); NULL: all B
    int n_rows = 0;
    DeltaAct act;
    // nq tokens per sequence in one launch (inputs [B][nq][H][...]): the state is read once
    // from chain[0][b] and the state after token t is stored to chain[t + 1][b] ([nq+1][B])
    int nq = 1;
    const int32_t *chain = nullptr;
    CopySkip skip;  // fault injection (tests only); inactive by default
};
cudaError_t launch_delta_decode(const DeltaDecodeArgs &a, cudaStream_t s);
bool delta_decode_supported(int dk, int dv);
uint32_t delta_decode_read_errors(bool clear);

struct AttnDecodeArgs {
    bool swa;
    int window;
    int ring_pages;  // SWA ring size in pages (>= ceil((window + nq - 1) / page_tokens))
    int nq = 1;      // new tokens per sequence (1: decode step; more: verification pass)
    const int32_t *rows = nullptr;  // batch rows to run (device, n_rows of them); NULL: all B
    int n_rows = 0;
    int B, Hq, Hkv, d, page_tokens;
    const void *q, *new_k, *new_v;
    void *k_pool, *v_pool;
    int n_pages;
    const int32_t *page_table;
    int max_pages;
    const int32_t *seq_lens;
    int max_seq_len;
    void *o;
    void *workspace;
    size_t ws_bytes;
    CopySkip skip;  // fault injection (tests only); inactive by default
};
struct AttnPlan {
    int n_splits;         // key ranges per (sequence, kv-head)
    int pages_per_split;
    int n_ctas;           // grid size: one CTA per (sequence, kv-head, key range)
    size_t ws_bytes;
};
AttnPlan attn_decode_plan(bool swa, int window, int B, int Hq, int Hkv, int d, int page_tokens,
                          int max_seq_len, int nq);
cudaError_t launch_attn_decode(const AttnDecodeArgs &a, cudaStream_t s);
bool attn_decode_supported(int d, int page_tokens, int group, int nq);
uint32_t attn_decode_read_errors(bool clear);

struct DeltaPrefillArgs {
    int kind;
    int B, T, H, dk, dv;
    bool bf16;
    const void *q, *k, *v;
    const float *beta, *log_gate;
    float *state;
    int n_slots;
    const int32_t *slots;
    void *o;
    int chunk;
    float scale;
    DeltaAct act;  // fused input activations (tensor-core path only)
};
cudaError_t launch_delta_prefill(const DeltaPrefillArgs &a, cudaStream_t s);
bool delta_prefill_supported(int dk, int dv, bool bf16, int chunk);
uint32_t delta_prefill_read_errors(bool clear);
// FA / SWA prefill of a prompt into the paged cache (attn_prefill_tc.cu)
struct AttnPrefillArgs {
    bool swa;
    int window;
    int B, T, Hq, Hkv, d, page_tokens;
    const void *q, *k, *v;
    void *k_pool, *v_pool;
    int n_pages;
    const int32_t *page_table;
    int max_pages;
    void *o;
    // cached prefix per sequence (device [B], multiples of page_tokens; NULL: none): token t
    // sits at position prefix_lens[b] + t and also attends the cached keys (tcgen05 path)
    const int32_t *prefix_lens = nullptr;
};
bool attn_prefill_supported(int d, int page_tokens, int group);
cudaError_t launch_attn_prefill(const AttnPrefillArgs &a, cudaStream_t s);
// the tcgen05 kernel (d = 64 or 128) behind launch_attn_prefill
bool attn_prefill_tc_supported(int d, int page_tokens, int group);
cudaError_t launch_attn_prefill_tc(const AttnPrefillArgs &a, cudaStream_t s);
uint32_t attn_prefill_tc_read_errors(bool clear);

// two-pass tensor-core path (bf16, d_k = d_v = 128, chunk 64): a chunk-parallel pass writes one
// record per chunk to a workspace, a scan pass carries the state through the chunks
struct PrefillScanArgs {
    const void *q, *k, *v;
    const float *beta, *log_gate;
    float *state;
    const int32_t *slots;
    int n_slots;
    void *o;
    int B, T, H;
    float scale;
    void *ws;         // records [B*H][n_seg][record bytes]
    int chunk_begin;  // first chunk of this segment
    int n_seg;        // chunks in this segment
    DeltaAct act;     // fused input activations
    int prefetch_stride = 0;  // prep: CTA i prefetches the inputs of CTA i + stride into L2
};
bool delta_prefill_scan_supported(int dk, int dv, bool bf16, int chunk);
size_t delta_prefill_scan_record_bytes();
// Runs the sequence in segments of as many chunks as ws_bytes holds for all B*H heads
// (cudaErrorInvalidValue if not even one chunk fits or ws is not 16-byte aligned).
cudaError_t launch_delta_prefill_scan(const DeltaPrefillArgs &a, void *ws, size_t ws_bytes,
                                      cudaStream_t s);
uint32_t delta_prefill_scan_read_errors(bool clear);


}  // namespace hmd

// C ABI of libhmd.so: argument validation, the recurrent-state and paged-KV caches, and the
// per-layer placement dispatcher. Every check here runs on the host before anything is
// launched, so a rejected call leaves device memory untouched.
//
// A placement picks one of four mixers per layer and can change between requests without
// reloading weights ("Super Apriel: One Checkpoint, Many Speeds", abstract; gist.science
// technical summary, section 2d). Here every layer's caches stay registered in the handles for
// their whole life, so a switch is a different placement array: nothing is copied.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <map>
#include <mutex>
#include <vector>

#include "kernels.h"
#include "../../include/hmd.h"

struct hmd_state_cache {
    int n_layers, slots, H, dk, dv;
    float *base;
    size_t layer_elems;
};

struct hmd_batch_plan {
    int n_layers, B;
    int32_t *rows_dev;             // [n_layers][B]: per layer, the rows of each kind in turn
    std::vector<int32_t> rows;     // host copy
    std::vector<int32_t> offsets;  // [n_layers][5]: kind k's rows are [offsets[k], offsets[k+1])
};

struct hmd_kv_cache {
    int n_layers, n_pools, n_pages, Hkv, d, page_tokens;
    std::vector<int32_t> layer_pool;
    std::vector<void *> k_pools, v_pools;
};

namespace {

thread_local hmd_status_t t_last = HMD_OK;

hmd_status_t fail(hmd_status_t s) {
    t_last = s;
    return s;
}

hmd_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? HMD_OK : fail(HMD_ERR_CUDA); }

// armed fault injections of this host thread (hmd_test_arm_copy_skip), one per test kernel
thread_local hmd::CopySkip t_skip[2];

cudaStream_t as_stream(hmd_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hmd_status_t check_delta_decode(hmd_kind_t kind, int B, int H, int dk, int dv, hmd_dtype_t dtype,
                                const void *q, const void *k, const void *v, const float *beta,
                                const float *log_gate, const float *state, int n_slots,
                                const void *o) {
    if (kind != HMD_GDN && kind != HMD_KDA) return HMD_ERR_ARG;
    if (dtype != HMD_F32 && dtype != HMD_BF16) return HMD_ERR_DTYPE;
    if (B < 0 || H < 1 || dk < 1 || dv < 1 || n_slots < 0) return HMD_ERR_SHAPE;
    if (B == 0) return HMD_OK;
    if (!q || !k || !v || !beta || !log_gate || !state || !o) return HMD_ERR_ARG;
    if (!hmd::delta_decode_supported(dk, dv)) return HMD_ERR_UNSUPPORTED;
    if (!aligned16(state) || !aligned16(o) || !aligned16(v)) return HMD_ERR_ARG;
    return HMD_OK;
}

}  // namespace

namespace hmd {
hmd_status_t record_status(hmd_status_t s) { return s == HMD_OK ? s : fail(s); }

CopySkip take_copy_skip(int kernel) {
    const CopySkip c = t_skip[kernel];
    t_skip[kernel] = CopySkip{};
    return c;
}
}  // namespace hmd

extern "C" {

hmd_status_t hmd_test_arm_copy_skip(hmd_test_kernel_t kernel, int cta, uint64_t wait_ns) {
    if ((kernel != HMD_TEST_DELTA_DECODE && kernel != HMD_TEST_ATTN_SPLIT) || cta < -1 ||
        wait_ns < 1000 || wait_ns > 2000000000ull)
        return fail(HMD_ERR_ARG);
    if (cta == -1) {  // disarm
        t_skip[kernel] = hmd::CopySkip{};
        return HMD_OK;
    }
    t_skip[kernel].cta = cta;
    t_skip[kernel].wait_ns = wait_ns;
    return HMD_OK;
}

const char *hmd_version(void) { return "hmd 0.1 (sm_100a)"; }

const char *hmd_status_string(hmd_status_t s) {
    switch (s) {
        case HMD_OK: return "ok";
        case HMD_ERR_ARG: return "invalid argument";
        case HMD_ERR_SHAPE: return "inconsistent shape";
        case HMD_ERR_DTYPE: return "unsupported dtype";
        case HMD_ERR_OOM: return "out of device memory";
        case HMD_ERR_CUDA: return "CUDA error";
        case HMD_ERR_UNSUPPORTED: return "unsupported configuration";
        case HMD_ERR_DEVICE_CHECK: return "device-side check fired";
    }
    return "unknown status";
}

hmd_status_t hmd_last_error(void) {
    const hmd_status_t s = t_last;
    t_last = HMD_OK;
    return s;
}

hmd_status_t hmd_device_errors(hmd_stream_t stream, uint32_t *bits, int clear) {
    if (!bits) return fail(HMD_ERR_ARG);
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return fail(HMD_ERR_CUDA);
    *bits = hmd::delta_decode_read_errors(clear != 0) | hmd::attn_decode_read_errors(clear != 0) |
            hmd::delta_prefill_read_errors(clear != 0) | hmd::delta_prefill_scan_read_errors(clear != 0) |
            hmd::attn_prefill_tc_read_errors(clear != 0);
    return HMD_OK;
}

// ---- delta-rule mixers -------------------------------------------------------------------

}  // extern "C"

namespace {
// delta_rule_decode_to over the batch rows `rows` (device, n_rows; NULL: every row of B).
hmd_status_t delta_run(hmd_kind_t kind, int B, int H, int dk, int dv, hmd_dtype_t dtype,
                       const void *q, const void *k, const void *v, const float *beta,
                       const float *log_gate, float *state, int n_slots, const int32_t *slots,
                       const int32_t *dst_slots, void *o, float scale, const int32_t *rows,
                       int n_rows, hmd_stream_t stream, const hmd_delta_act_t *act = nullptr,
                       int nq = 1, const int32_t *chain = nullptr) {
    const hmd_status_t st = check_delta_decode(kind, B, H, dk, dv, dtype, q, k, v, beta, log_gate,
                                               state, n_slots, o);
    if (st != HMD_OK) return fail(st);
    if (B == 0 || (rows && n_rows == 0)) return HMD_OK;
    if (!slots && n_slots < B) return fail(HMD_ERR_SHAPE);
    hmd::DeltaDecodeArgs a{};
    a.kind = kind; a.B = B; a.H = H; a.dk = dk; a.dv = dv; a.bf16 = dtype == HMD_BF16;
    a.q = q; a.k = k; a.v = v; a.beta = beta; a.log_gate = log_gate; a.state = state;
    a.n_slots = n_slots; a.slots = slots; a.dst_slots = dst_slots; a.o = o; a.scale = scale;
    a.rows = rows; a.n_rows = n_rows;
    if (act) {
        if (!act->A_log || !act->dt_bias || !(act->l2_eps >= 0.f)) return fail(HMD_ERR_ARG);
        a.act.A_log = act->A_log; a.act.dt_bias = act->dt_bias; a.act.eps = act->l2_eps;
    }
    a.nq = nq; a.chain = chain;
    a.skip = hmd::take_copy_skip(HMD_TEST_DELTA_DECODE);
    return from_cuda(hmd::launch_delta_decode(a, as_stream(stream)));
}
}  // namespace

extern "C" {

hmd_status_t delta_rule_decode_to(hmd_kind_t kind, int B, int H, int dk, int dv,
                                  hmd_dtype_t dtype, const void *q, const void *k, const void *v,
                                  const float *beta, const float *log_gate, float *state,
                                  int n_slots, const int32_t *slots, const int32_t *dst_slots,
                                  void *o, float scale, hmd_stream_t stream) {
    return delta_run(kind, B, H, dk, dv, dtype, q, k, v, beta, log_gate, state, n_slots, slots,
                     dst_slots, o, scale, nullptr, 0, stream);
}

hmd_status_t delta_rule_decode_act(hmd_kind_t kind, int B, int H, int dk, int dv,
                                   hmd_dtype_t dtype, const void *q_raw, const void *k_raw,
                                   const void *v, const float *beta_logit,
                                   const float *gate_logit, const hmd_delta_act_t *act,
                                   float *state, int n_slots, const int32_t *slots,
                                   const int32_t *dst_slots, void *o, float scale,
                                   hmd_stream_t stream) {
    if (!act) return fail(HMD_ERR_ARG);
    return delta_run(kind, B, H, dk, dv, dtype, q_raw, k_raw, v, beta_logit, gate_logit, state,
                     n_slots, slots, dst_slots, o, scale, nullptr, 0, stream, act);
}

hmd_status_t delta_rule_decode_chain(hmd_kind_t kind, int n_q, int B, int H, int dk, int dv,
                                     hmd_dtype_t dtype, const void *q, const void *k,
                                     const void *v, const float *beta, const float *log_gate,
                                     const hmd_delta_act_t *act, float *state, int n_slots,
                                     const int32_t *chain, void *o, float scale,
                                     hmd_stream_t stream) {
    if (n_q < 1) return fail(HMD_ERR_SHAPE);
    if (!chain && B > 0) return fail(HMD_ERR_ARG);
    return delta_run(kind, B, H, dk, dv, dtype, q, k, v, beta, log_gate, state, n_slots, nullptr,
                     nullptr, o, scale, nullptr, 0, stream, act, n_q, chain);
}

hmd_status_t delta_rule_decode(hmd_kind_t kind, int B, int H, int dk, int dv, hmd_dtype_t dtype,
                               const void *q, const void *k, const void *v, const float *beta,
                               const float *log_gate, float *state, int n_slots,
                               const int32_t *slots, void *o, float scale, hmd_stream_t stream) {
    return delta_rule_decode_to(kind, B, H, dk, dv, dtype, q, k, v, beta, log_gate, state,
                                n_slots, slots, nullptr, o, scale, stream);
}

}  // extern "C"

namespace {

// Scratch of the two-pass prefill when the caller passes none: a stream-ordered allocation from
// a library-owned pool per device that keeps up to kPrefillPoolKeep bytes cached between calls.
constexpr size_t kPrefillWsCap = size_t(1) << 30;   // per call: longer inputs run in segments
constexpr uint64_t kPrefillPoolKeep = uint64_t(1) << 30;

cudaMemPool_t prefill_pool() {
    static std::mutex mu;
    static std::map<int, cudaMemPool_t> pools;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    auto it = pools.find(dev);
    if (it != pools.end()) return it->second;
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
    uint64_t keep = kPrefillPoolKeep;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    pools[dev] = pool;
    return pool;
}

hmd_status_t check_prefill(hmd_kind_t kind, int B, int T, int H, int dk, int dv,
                           hmd_dtype_t dtype, const void *q, const void *k, const void *v,
                           const float *beta, const float *log_gate, const float *state,
                           int n_slots, const int32_t *slots, const void *o, int chunk) {
    if (kind != HMD_GDN && kind != HMD_KDA) return HMD_ERR_ARG;
    if (dtype != HMD_F32 && dtype != HMD_BF16) return HMD_ERR_DTYPE;
    if (B < 0 || T < 0 || H < 1 || dk < 1 || dv < 1 || n_slots < 0 || chunk < 1)
        return HMD_ERR_SHAPE;
    if (B == 0 || T == 0) return HMD_OK;
    if (!q || !k || !v || !beta || !log_gate || !state || !o) return HMD_ERR_ARG;
    if (!slots && n_slots < B) return HMD_ERR_SHAPE;
    if (!hmd::delta_prefill_supported(dk, dv, dtype == HMD_BF16, chunk)) return HMD_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state) ||
        !aligned16(log_gate))
        return HMD_ERR_ARG;
    return HMD_OK;
}

hmd::DeltaPrefillArgs prefill_args(hmd_kind_t kind, int B, int T, int H, int dk, int dv,
                                   hmd_dtype_t dtype, const void *q, const void *k, const void *v,
                                   const float *beta, const float *log_gate, float *state,
                                   int n_slots, const int32_t *slots, void *o, int chunk,
                                   float scale) {
    hmd::DeltaPrefillArgs a{};
    a.kind = kind; a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.bf16 = dtype == HMD_BF16;
    a.q = q; a.k = k; a.v = v; a.beta = beta; a.log_gate = log_gate; a.state = state;
    a.n_slots = n_slots; a.slots = slots; a.o = o; a.chunk = chunk; a.scale = scale;
    return a;
}

// bytes of one chunk record for every (sequence, head): the smallest usable workspace
size_t prefill_min_ws(int B, int H) {
    return (size_t)B * H * hmd::delta_prefill_scan_record_bytes();
}

}  // namespace

extern "C" {

size_t delta_rule_prefill_workspace_size(hmd_kind_t kind, int B, int T, int H, int dk, int dv,
                                         hmd_dtype_t dtype, int chunk) {
    (void)kind;
    if (B < 1 || T < 1 || H < 1 || chunk < 1) return 0;
    if (!hmd::delta_prefill_scan_supported(dk, dv, dtype == HMD_BF16, chunk)) return 0;
    const size_t n_chunks = (size_t)(T + chunk - 1) / chunk;
    return prefill_min_ws(B, H) * n_chunks;
}

hmd_status_t delta_rule_prefill_chunked_ws(hmd_kind_t kind, int B, int T, int H, int dk, int dv,
                                           hmd_dtype_t dtype, const void *q, const void *k,
                                           const void *v, const float *beta,
                                           const float *log_gate, float *state, int n_slots,
                                           const int32_t *slots, void *o, int chunk, float scale,
                                           void *workspace, size_t ws_bytes,
                                           hmd_stream_t stream) {
    const hmd_status_t st = check_prefill(kind, B, T, H, dk, dv, dtype, q, k, v, beta, log_gate,
                                          state, n_slots, slots, o, chunk);
    if (st != HMD_OK) return fail(st);
    if (B == 0 || T == 0) return HMD_OK;
    const hmd::DeltaPrefillArgs a = prefill_args(kind, B, T, H, dk, dv, dtype, q, k, v, beta,
                                                 log_gate, state, n_slots, slots, o, chunk, scale);
    if (!hmd::delta_prefill_scan_supported(dk, dv, dtype == HMD_BF16, chunk))
        return from_cuda(hmd::launch_delta_prefill(a, as_stream(stream)));
    if (!workspace || !aligned16(workspace)) return fail(HMD_ERR_ARG);
    if (ws_bytes < prefill_min_ws(B, H)) return fail(HMD_ERR_SHAPE);
    return from_cuda(hmd::launch_delta_prefill_scan(a, workspace, ws_bytes, as_stream(stream)));
}

}  // extern "C"

namespace {
hmd_status_t prefill_pooled(hmd_kind_t kind, int B, int T, int H, int dk, int dv,
                            hmd_dtype_t dtype, const void *q, const void *k, const void *v,
                            const float *beta, const float *log_gate, float *state, int n_slots,
                            const int32_t *slots, void *o, int chunk, float scale,
                            const hmd_delta_act_t *act, hmd_stream_t stream) {
    const hmd_status_t st = check_prefill(kind, B, T, H, dk, dv, dtype, q, k, v, beta, log_gate,
                                          state, n_slots, slots, o, chunk);
    if (st != HMD_OK) return fail(st);
    if (act) {
        if (!act->A_log || !act->dt_bias || !(act->l2_eps >= 0.f)) return fail(HMD_ERR_ARG);
        // the fused activations live in the tensor-core path's chunk-parallel pass
        if (!hmd::delta_prefill_scan_supported(dk, dv, dtype == HMD_BF16, chunk))
            return fail(HMD_ERR_UNSUPPORTED);
    }
    if (B == 0 || T == 0) return HMD_OK;
    hmd::DeltaPrefillArgs a = prefill_args(kind, B, T, H, dk, dv, dtype, q, k, v, beta,
                                           log_gate, state, n_slots, slots, o, chunk, scale);
    if (act) {
        a.act.A_log = act->A_log; a.act.dt_bias = act->dt_bias; a.act.eps = act->l2_eps;
    }
    if (!hmd::delta_prefill_scan_supported(dk, dv, dtype == HMD_BF16, chunk))
        return from_cuda(hmd::launch_delta_prefill(a, as_stream(stream)));
    const size_t full = delta_rule_prefill_workspace_size(kind, B, T, H, dk, dv, dtype, chunk);
    const size_t bytes = full <= kPrefillWsCap ? full : std::max(prefill_min_ws(B, H), kPrefillWsCap);
    cudaMemPool_t pool = prefill_pool();
    if (!pool) return fail(HMD_ERR_CUDA);
    const cudaStream_t s = as_stream(stream);
    void *ws = nullptr;
    if (cudaMallocFromPoolAsync(&ws, bytes, pool, s) != cudaSuccess) {
        cudaGetLastError();
        return fail(HMD_ERR_OOM);
    }
    const cudaError_t e = hmd::launch_delta_prefill_scan(a, ws, bytes, s);
    const cudaError_t f = cudaFreeAsync(ws, s);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(f);
}
}  // namespace

extern "C" {

hmd_status_t delta_rule_prefill_chunked(hmd_kind_t kind, int B, int T, int H, int dk, int dv,
                                        hmd_dtype_t dtype, const void *q, const void *k,
                                        const void *v, const float *beta, const float *log_gate,
                                        float *state, int n_slots, const int32_t *slots, void *o,
                                        int chunk, float scale, hmd_stream_t stream) {
    return prefill_pooled(kind, B, T, H, dk, dv, dtype, q, k, v, beta, log_gate, state, n_slots,
                          slots, o, chunk, scale, nullptr, stream);
}

hmd_status_t delta_rule_prefill_chunked_act(hmd_kind_t kind, int B, int T, int H, int dk, int dv,
                                            hmd_dtype_t dtype, const void *q_raw,
                                            const void *k_raw, const void *v,
                                            const float *beta_logit, const float *gate_logit,
                                            const hmd_delta_act_t *act, float *state,
                                            int n_slots, const int32_t *slots, void *o, int chunk,
                                            float scale, hmd_stream_t stream) {
    if (!act) return fail(HMD_ERR_ARG);
    return prefill_pooled(kind, B, T, H, dk, dv, dtype, q_raw, k_raw, v, beta_logit, gate_logit,
                          state, n_slots, slots, o, chunk, scale, act, stream);
}

// ---- attention mixers --------------------------------------------------------------------

hmd_status_t attn_prefill_ext(hmd_kind_t kind, int window, int B, int T, int Hq, int Hkv, int d,
                              int page_tokens, const void *q, const void *k, const void *v,
                              const int32_t *prefix_lens, int max_prefix, void *k_pool,
                              void *v_pool, int n_pages, const int32_t *page_table, int max_pages,
                              void *o, hmd_stream_t stream) {
    if (kind != HMD_FA && kind != HMD_SWA) return fail(HMD_ERR_ARG);
    if (kind == HMD_SWA && window < 1) return fail(HMD_ERR_ARG);
    if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || d < 1 || page_tokens < 1 || n_pages < 1 ||
        max_pages < 1 || max_prefix < 0)
        return fail(HMD_ERR_SHAPE);
    if (Hq % Hkv) return fail(HMD_ERR_SHAPE);
    if (prefix_lens && max_prefix % page_tokens) return fail(HMD_ERR_SHAPE);
    if (B == 0 || T == 0) return HMD_OK;
    if (!q || !k || !v || !k_pool || !v_pool || !page_table || !o) return fail(HMD_ERR_ARG);
    if (!hmd::attn_prefill_supported(d, page_tokens, Hq / Hkv)) return fail(HMD_ERR_UNSUPPORTED);
    const long long span = (long long)(prefix_lens ? max_prefix : 0) + T;
    const long long need = kind == HMD_SWA ? (window + page_tokens - 1) / page_tokens
                                           : (span + page_tokens - 1) / page_tokens;
    if (max_pages < need) return fail(HMD_ERR_SHAPE);
    if ((long long)n_pages * Hkv * page_tokens >= (1LL << 31)) return fail(HMD_ERR_UNSUPPORTED);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(k_pool) ||
        !aligned16(v_pool))
        return fail(HMD_ERR_ARG);
    hmd::AttnPrefillArgs a{};
    a.swa = kind == HMD_SWA; a.window = window; a.B = B; a.T = T; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
    a.page_tokens = page_tokens; a.q = q; a.k = k; a.v = v; a.k_pool = k_pool; a.v_pool = v_pool;
    a.n_pages = n_pages; a.page_table = page_table; a.max_pages = max_pages; a.o = o;
    a.prefix_lens = prefix_lens;
    return from_cuda(hmd::launch_attn_prefill(a, as_stream(stream)));
}

hmd_status_t attn_prefill(hmd_kind_t kind, int window, int B, int T, int Hq, int Hkv, int d,
                          int page_tokens, const void *q, const void *k, const void *v,
                          void *k_pool, void *v_pool, int n_pages, const int32_t *page_table,
                          int max_pages, void *o, hmd_stream_t stream) {
    return attn_prefill_ext(kind, window, B, T, Hq, Hkv, d, page_tokens, q, k, v, nullptr, 0,
                            k_pool, v_pool, n_pages, page_table, max_pages, o, stream);
}

size_t attn_verify_workspace_size(hmd_kind_t kind, int window, int n_q, int B, int Hq, int Hkv,
                                  int d, int page_tokens, int max_seq_len) {
    if (B < 1 || Hq < 1 || Hkv < 1 || d < 1 || max_seq_len < 1 || n_q < 1) return 16;
    const hmd::AttnPlan pl = hmd::attn_decode_plan(kind == HMD_SWA, window, B, Hq, Hkv, d,
                                                   page_tokens, max_seq_len, n_q);
    return pl.ws_bytes < 16 ? 16 : pl.ws_bytes;
}

size_t attn_decode_workspace_size(hmd_kind_t kind, int window, int B, int Hq, int Hkv, int d,
                                  int page_tokens, int max_seq_len) {
    return attn_verify_workspace_size(kind, window, 1, B, Hq, Hkv, d, page_tokens, max_seq_len);
}

}  // extern "C"

namespace {
// attn_verify over the batch rows `rows` (device, n_rows of them; NULL: every row of B).
hmd_status_t attn_run(hmd_kind_t kind, int window, int ring_pages, int n_q, int B, int Hq,
                      int Hkv, int d, int page_tokens, const void *q, const void *new_k,
                      const void *new_v, void *k_pool, void *v_pool, int n_pages,
                      const int32_t *page_table, int max_pages, const int32_t *seq_lens,
                      int max_seq_len, void *o, void *workspace, size_t ws_bytes,
                      const int32_t *rows, int n_rows, hmd_stream_t stream) {
    if (kind != HMD_FA && kind != HMD_SWA) return fail(HMD_ERR_ARG);
    if (kind == HMD_SWA && window < 1) return fail(HMD_ERR_ARG);
    if (B < 0 || n_q < 1 || Hq < 1 || Hkv < 1 || d < 1 || page_tokens < 1 || n_pages < 1 ||
        max_pages < 1 || max_seq_len < 1)
        return fail(HMD_ERR_SHAPE);
    if (Hq % Hkv) return fail(HMD_ERR_SHAPE);
    if (B == 0) return HMD_OK;
    if (!q || !new_k || !new_v || !k_pool || !v_pool || !page_table || !seq_lens || !o ||
        !workspace)
        return fail(HMD_ERR_ARG);
    if (!hmd::attn_decode_supported(d, page_tokens, Hq / Hkv, n_q)) return fail(HMD_ERR_UNSUPPORTED);
    const long long seq_pages = ((long long)max_seq_len + page_tokens - 1) / page_tokens;
    long long need = seq_pages;  // FA: the table covers the longest sequence
    if (kind == HMD_SWA) {
        // the ring must hold every key of the n_q rows at once: window + n_q - 1 positions
        const long long min_ring = ((long long)window + n_q - 1 + page_tokens - 1) / page_tokens;
        if (ring_pages < min_ring) return fail(HMD_ERR_SHAPE);
        need = ring_pages < seq_pages ? ring_pages : seq_pages;
    }
    if (max_pages < need) return fail(HMD_ERR_SHAPE);
    if ((long long)n_pages * Hkv * page_tokens >= (1LL << 31)) return fail(HMD_ERR_UNSUPPORTED);
    if (!aligned16(q) || !aligned16(new_k) || !aligned16(new_v) || !aligned16(k_pool) ||
        !aligned16(v_pool) || !aligned16(workspace))
        return fail(HMD_ERR_ARG);
    const hmd::AttnPlan pl = hmd::attn_decode_plan(kind == HMD_SWA, window, rows ? n_rows : B, Hq,
                                                   Hkv, d, page_tokens, max_seq_len, n_q);
    if (ws_bytes < pl.ws_bytes) return fail(HMD_ERR_SHAPE);
    hmd::AttnDecodeArgs a{};
    a.swa = kind == HMD_SWA; a.window = window; a.ring_pages = ring_pages; a.nq = n_q;
    a.rows = rows; a.n_rows = n_rows;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.d = d;
    a.page_tokens = page_tokens; a.q = q; a.new_k = new_k; a.new_v = new_v;
    a.k_pool = k_pool; a.v_pool = v_pool; a.n_pages = n_pages; a.page_table = page_table;
    a.max_pages = max_pages; a.seq_lens = seq_lens; a.max_seq_len = max_seq_len; a.o = o;
    a.workspace = workspace; a.ws_bytes = ws_bytes;
    a.skip = hmd::take_copy_skip(HMD_TEST_ATTN_SPLIT);
    return from_cuda(hmd::launch_attn_decode(a, as_stream(stream)));
}
}  // namespace

extern "C" {

hmd_status_t attn_verify(hmd_kind_t kind, int window, int ring_pages, int n_q, int B, int Hq,
                         int Hkv, int d, int page_tokens, const void *q, const void *new_k,
                         const void *new_v, void *k_pool, void *v_pool, int n_pages,
                         const int32_t *page_table, int max_pages, const int32_t *seq_lens,
                         int max_seq_len, void *o, void *workspace, size_t ws_bytes,
                         hmd_stream_t stream) {
    return attn_run(kind, window, ring_pages, n_q, B, Hq, Hkv, d, page_tokens, q, new_k, new_v,
                    k_pool, v_pool, n_pages, page_table, max_pages, seq_lens, max_seq_len, o,
                    workspace, ws_bytes, nullptr, 0, stream);
}

hmd_status_t attn_decode(hmd_kind_t kind, int window, int B, int Hq, int Hkv, int d,
                         int page_tokens, const void *q, const void *new_k, const void *new_v,
                         void *k_pool, void *v_pool, int n_pages, const int32_t *page_table,
                         int max_pages, const int32_t *seq_lens, int max_seq_len, void *o,
                         void *workspace, size_t ws_bytes, hmd_stream_t stream) {
    // the decode step is the one-token verification pass on the ring of ceil(window / 64) pages
    const int ring = (kind == HMD_SWA && window >= 1 && page_tokens >= 1)
                         ? (int)(((long long)window + page_tokens - 1) / page_tokens)
                         : 0;
    return attn_verify(kind, window, ring, 1, B, Hq, Hkv, d, page_tokens, q, new_k, new_v, k_pool,
                       v_pool, n_pages, page_table, max_pages, seq_lens, max_seq_len, o,
                       workspace, ws_bytes, stream);
}

// ---- caches ------------------------------------------------------------------------------

hmd_status_t state_cache_alloc(int n_layers, int slots, int H, int dk, int dv,
                               hmd_stream_t stream, hmd_state_cache_t **out) {
    if (!out) return fail(HMD_ERR_ARG);
    *out = nullptr;
    if (n_layers < 1 || slots < 1 || H < 1 || dk < 1 || dv < 1) return fail(HMD_ERR_SHAPE);
    auto *c = new (std::nothrow) hmd_state_cache{n_layers, slots, H, dk, dv, nullptr, 0};
    if (!c) return fail(HMD_ERR_OOM);
    c->layer_elems = (size_t)slots * H * dk * dv;
    const size_t bytes = c->layer_elems * n_layers * sizeof(float);
    cudaStream_t s = as_stream(stream);
    if (cudaMallocAsync(reinterpret_cast<void **>(&c->base), bytes, s) != cudaSuccess) {
        cudaGetLastError();
        delete c;
        return fail(HMD_ERR_OOM);
    }
    if (cudaMemsetAsync(c->base, 0, bytes, s) != cudaSuccess) {
        cudaFreeAsync(c->base, s);
        delete c;
        return fail(HMD_ERR_CUDA);
    }
    *out = c;
    return HMD_OK;
}

hmd_status_t state_cache_free(hmd_state_cache_t *c, hmd_stream_t stream) {
    if (!c) return fail(HMD_ERR_ARG);
    const cudaError_t e = cudaFreeAsync(c->base, as_stream(stream));
    delete c;
    return from_cuda(e);
}

hmd_status_t state_cache_layer(hmd_state_cache_t *c, int layer, float **out) {
    if (!c || !out) return fail(HMD_ERR_ARG);
    if (layer < 0 || layer >= c->n_layers) return fail(HMD_ERR_ARG);
    *out = c->base + c->layer_elems * layer;
    return HMD_OK;
}

hmd_status_t state_cache_reset(hmd_state_cache_t *c, int layer, const int32_t *slot_ids, int n,
                               const float *init, hmd_stream_t stream) {
    if (!c || (n > 0 && !slot_ids)) return fail(HMD_ERR_ARG);
    if (layer < 0 || layer >= c->n_layers || n < 0) return fail(HMD_ERR_ARG);
    for (int i = 0; i < n; ++i)
        if (slot_ids[i] < 0 || slot_ids[i] >= c->slots) return fail(HMD_ERR_ARG);
    const size_t per = (size_t)c->H * c->dk * c->dv;
    float *blk = c->base + c->layer_elems * layer;
    cudaStream_t s = as_stream(stream);
    for (int i = 0; i < n; ++i) {
        float *dst = blk + per * slot_ids[i];
        const cudaError_t e = init ? cudaMemcpyAsync(dst, init + per * i, per * sizeof(float),
                                                     cudaMemcpyDeviceToDevice, s)
                                   : cudaMemsetAsync(dst, 0, per * sizeof(float), s);
        if (e != cudaSuccess) return fail(HMD_ERR_CUDA);
    }
    return HMD_OK;
}

hmd_status_t state_cache_save(hmd_state_cache_t *c, int layer, const int32_t *slot_ids, int n,
                              float *out, hmd_stream_t stream) {
    if (!c || (n > 0 && (!slot_ids || !out))) return fail(HMD_ERR_ARG);
    if (layer < 0 || layer >= c->n_layers || n < 0) return fail(HMD_ERR_ARG);
    for (int i = 0; i < n; ++i)
        if (slot_ids[i] < 0 || slot_ids[i] >= c->slots) return fail(HMD_ERR_ARG);
    const size_t per = (size_t)c->H * c->dk * c->dv;
    const float *blk = c->base + c->layer_elems * layer;
    cudaStream_t s = as_stream(stream);
    for (int i = 0; i < n; ++i) {  // one device-to-device copy per slot
        if (cudaMemcpyAsync(out + per * i, blk + per * slot_ids[i], per * sizeof(float),
                            cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return fail(HMD_ERR_CUDA);
    }
    return HMD_OK;
}

hmd_status_t kv_cache_alloc(int n_layers, const int32_t *layer_pool, int n_pools, int n_pages,
                            int Hkv, int d, int page_tokens, hmd_stream_t stream,
                            hmd_kv_cache_t **out) {
    if (!out || !layer_pool) return fail(HMD_ERR_ARG);
    *out = nullptr;
    if (n_layers < 1 || n_pools < 0 || n_pages < 1 || Hkv < 1 || d < 1 || page_tokens < 1)
        return fail(HMD_ERR_SHAPE);
    for (int l = 0; l < n_layers; ++l)
        if (layer_pool[l] < -1 || layer_pool[l] >= n_pools) return fail(HMD_ERR_ARG);
    auto *c = new (std::nothrow) hmd_kv_cache;
    if (!c) return fail(HMD_ERR_OOM);
    c->n_layers = n_layers; c->n_pools = n_pools; c->n_pages = n_pages; c->Hkv = Hkv; c->d = d;
    c->page_tokens = page_tokens;
    c->layer_pool.assign(layer_pool, layer_pool + n_layers);
    const size_t bytes = (size_t)n_pages * Hkv * page_tokens * d * 2;
    cudaStream_t s = as_stream(stream);
    for (int i = 0; i < n_pools; ++i) {
        void *kp = nullptr, *vp = nullptr;
        if (cudaMallocAsync(&kp, bytes, s) != cudaSuccess ||
            cudaMallocAsync(&vp, bytes, s) != cudaSuccess) {
            cudaGetLastError();
            if (kp) cudaFreeAsync(kp, s);
            for (size_t j = 0; j < c->k_pools.size(); ++j) {
                cudaFreeAsync(c->k_pools[j], s);
                cudaFreeAsync(c->v_pools[j], s);
            }
            delete c;
            return fail(HMD_ERR_OOM);
        }
        cudaMemsetAsync(kp, 0, bytes, s);
        cudaMemsetAsync(vp, 0, bytes, s);
        c->k_pools.push_back(kp);
        c->v_pools.push_back(vp);
    }
    *out = c;
    return HMD_OK;
}

hmd_status_t kv_cache_free(hmd_kv_cache_t *c, hmd_stream_t stream) {
    if (!c) return fail(HMD_ERR_ARG);
    cudaError_t e = cudaSuccess;
    for (size_t j = 0; j < c->k_pools.size(); ++j) {
        if (cudaFreeAsync(c->k_pools[j], as_stream(stream)) != cudaSuccess) e = cudaErrorUnknown;
        if (cudaFreeAsync(c->v_pools[j], as_stream(stream)) != cudaSuccess) e = cudaErrorUnknown;
    }
    delete c;
    return from_cuda(e);
}

hmd_status_t kv_cache_layer(hmd_kv_cache_t *c, int layer, void **k_pool, void **v_pool) {
    if (!c || !k_pool || !v_pool) return fail(HMD_ERR_ARG);
    if (layer < 0 || layer >= c->n_layers) return fail(HMD_ERR_ARG);
    const int p = c->layer_pool[layer];
    if (p < 0) return fail(HMD_ERR_ARG);
    *k_pool = c->k_pools[p];
    *v_pool = c->v_pools[p];
    return HMD_OK;
}

// ---- the placement dispatcher -------------------------------------------------------------

hmd_status_t mixer_decode_step(const int8_t *placement, int n_layers, int layer,
                               const hmd_decode_io_t *io, hmd_state_cache_t *sc,
                               hmd_kv_cache_t *kc, void *workspace, size_t ws_bytes,
                               hmd_stream_t stream) {
    if (!placement || !io || n_layers < 1 || layer < 0 || layer >= n_layers)
        return fail(HMD_ERR_ARG);
    const int kind = placement[layer];
    switch (kind) {
        case HMD_GDN:
        case HMD_KDA: {
            if (!sc || layer >= sc->n_layers) return fail(HMD_ERR_ARG);
            if (io->H != sc->H || io->d != sc->dk || io->d != sc->dv) return fail(HMD_ERR_SHAPE);
            if (!io->slots && io->B > sc->slots) return fail(HMD_ERR_SHAPE);
            float *state = sc->base + sc->layer_elems * layer;
            const float *lg = kind == HMD_GDN ? io->log_gate_scalar : io->log_gate_channel;
            return delta_rule_decode(static_cast<hmd_kind_t>(kind), io->B, io->H, io->d, io->d,
                                     io->dtype, io->q, io->k, io->v, io->beta, lg, state,
                                     sc->slots, io->slots, io->o, io->scale, stream);
        }
        case HMD_FA:
        case HMD_SWA: {
            if (!kc || layer >= kc->n_layers || kc->layer_pool[layer] < 0) return fail(HMD_ERR_ARG);
            if (io->dtype != HMD_BF16) return fail(HMD_ERR_DTYPE);
            if (io->Hkv != kc->Hkv || io->d != kc->d) return fail(HMD_ERR_SHAPE);
            const int p = kc->layer_pool[layer];
            return attn_decode(static_cast<hmd_kind_t>(kind), io->window, io->B, io->H, io->Hkv,
                               io->d, kc->page_tokens, io->q, io->k, io->v, kc->k_pools[p],
                               kc->v_pools[p], kc->n_pages, io->page_table, io->max_pages,
                               io->seq_lens, io->max_seq_len, io->o, workspace, ws_bytes, stream);
        }
        default:
            return fail(HMD_ERR_ARG);
    }
}

// ---- mixed placements in one batch -------------------------------------------------------

hmd_status_t hmd_group_sequences(int n_layers, int n_placements, const int8_t *placements, int B,
                                 const int32_t *seq_placement, int32_t *rows, int32_t *offsets) {
    if (!placements || !seq_placement || !rows || !offsets || n_layers < 1 || n_placements < 1 ||
        B < 1)
        return fail(HMD_ERR_ARG);
    for (int p = 0; p < n_placements * n_layers; ++p)
        if (placements[p] < HMD_FA || placements[p] > HMD_GDN) return fail(HMD_ERR_ARG);
    for (int b = 0; b < B; ++b)
        if (seq_placement[b] < 0 || seq_placement[b] >= n_placements) return fail(HMD_ERR_ARG);
    for (int l = 0; l < n_layers; ++l) {
        int32_t *r = rows + (size_t)l * B;
        int32_t *off = offsets + (size_t)l * 5;
        int n = 0;
        for (int kind = HMD_FA; kind <= HMD_GDN; ++kind) {
            off[kind] = n;
            for (int b = 0; b < B; ++b)
                if (placements[(size_t)seq_placement[b] * n_layers + l] == kind) r[n++] = b;
        }
        off[4] = n;
    }
    return HMD_OK;
}

hmd_status_t batch_plan_create(int n_layers, int n_placements, const int8_t *placements, int B,
                               const int32_t *seq_placement, hmd_stream_t stream,
                               hmd_batch_plan_t **out) {
    if (!out) return fail(HMD_ERR_ARG);
    *out = nullptr;
    std::vector<int32_t> rows((size_t)n_layers * (B > 0 ? B : 0)), offs((size_t)n_layers * 5);
    const hmd_status_t st = hmd_group_sequences(n_layers, n_placements, placements, B,
                                                seq_placement, rows.data(), offs.data());
    if (st != HMD_OK) return st;
    void *dev = nullptr;
    if (cudaMallocAsync(&dev, rows.size() * sizeof(int32_t), as_stream(stream)) != cudaSuccess) {
        cudaGetLastError();
        return fail(HMD_ERR_OOM);
    }
    // pageable source: the call returns once the host buffer has been staged
    if (cudaMemcpyAsync(dev, rows.data(), rows.size() * sizeof(int32_t), cudaMemcpyHostToDevice,
                        as_stream(stream)) != cudaSuccess) {
        cudaFreeAsync(dev, as_stream(stream));
        return fail(HMD_ERR_CUDA);
    }
    auto *pl = new (std::nothrow) hmd_batch_plan;
    if (!pl) {
        cudaFreeAsync(dev, as_stream(stream));
        return fail(HMD_ERR_OOM);
    }
    pl->n_layers = n_layers;
    pl->B = B;
    pl->rows_dev = static_cast<int32_t *>(dev);
    pl->rows = std::move(rows);
    pl->offsets = std::move(offs);
    *out = pl;
    return HMD_OK;
}

hmd_status_t batch_plan_free(hmd_batch_plan_t *plan, hmd_stream_t stream) {
    if (!plan) return HMD_OK;
    const cudaError_t e = cudaFreeAsync(plan->rows_dev, as_stream(stream));
    delete plan;
    return e == cudaSuccess ? HMD_OK : fail(HMD_ERR_CUDA);
}

hmd_status_t batch_plan_group(const hmd_batch_plan_t *plan, int layer, hmd_kind_t kind,
                              int *count, const int32_t **rows_host) {
    if (!plan || !count || layer < 0 || layer >= plan->n_layers || kind < HMD_FA ||
        kind > HMD_GDN)
        return fail(HMD_ERR_ARG);
    const int32_t *off = plan->offsets.data() + (size_t)layer * 5;
    *count = off[kind + 1] - off[kind];
    if (rows_host) *rows_host = plan->rows.data() + (size_t)layer * plan->B + off[kind];
    return HMD_OK;
}

size_t batch_plan_workspace_size(const hmd_batch_plan_t *plan, int window, int Hq, int Hkv, int d,
                                 int page_tokens, int max_seq_len) {
    size_t best = 16;
    if (!plan) return best;
    for (int l = 0; l < plan->n_layers; ++l) {
        const int32_t *off = plan->offsets.data() + (size_t)l * 5;
        for (int kind = HMD_FA; kind <= HMD_SWA; ++kind) {
            const int n = off[kind + 1] - off[kind];
            if (n > 0)
                best = std::max(best, attn_verify_workspace_size(static_cast<hmd_kind_t>(kind),
                                                                 window, 1, n, Hq, Hkv, d,
                                                                 page_tokens, max_seq_len));
        }
    }
    return best;
}

hmd_status_t mixer_decode_step_batch(const hmd_batch_plan_t *plan, int layer,
                                     const hmd_decode_io_t *const *io, hmd_state_cache_t *sc,
                                     hmd_kv_cache_t *kc, void *workspace, size_t ws_bytes,
                                     hmd_stream_t stream) {
    if (!plan || !io || layer < 0 || layer >= plan->n_layers) return fail(HMD_ERR_ARG);
    const int32_t *off = plan->offsets.data() + (size_t)layer * 5;
    const int32_t *rows = plan->rows_dev + (size_t)layer * plan->B;
    for (int kind = HMD_FA; kind <= HMD_GDN; ++kind) {
        const int n = off[kind + 1] - off[kind];
        if (n == 0) continue;
        const hmd_decode_io_t *x = io[kind];
        if (!x) return fail(HMD_ERR_ARG);
        if (x->B != plan->B) return fail(HMD_ERR_SHAPE);
        hmd_status_t st;
        if (kind == HMD_GDN || kind == HMD_KDA) {
            if (!sc || layer >= sc->n_layers) return fail(HMD_ERR_ARG);
            if (x->H != sc->H || x->d != sc->dk || x->d != sc->dv) return fail(HMD_ERR_SHAPE);
            if (!x->slots && x->B > sc->slots) return fail(HMD_ERR_SHAPE);
            float *state = sc->base + sc->layer_elems * layer;
            const float *lg = kind == HMD_GDN ? x->log_gate_scalar : x->log_gate_channel;
            st = delta_run(static_cast<hmd_kind_t>(kind), x->B, x->H, x->d, x->d, x->dtype, x->q,
                           x->k, x->v, x->beta, lg, state, sc->slots, x->slots, nullptr, x->o,
                           x->scale, rows + off[kind], n, stream);
        } else {
            if (!kc || layer >= kc->n_layers || kc->layer_pool[layer] < 0) return fail(HMD_ERR_ARG);
            if (x->dtype != HMD_BF16) return fail(HMD_ERR_DTYPE);
            if (x->Hkv != kc->Hkv || x->d != kc->d) return fail(HMD_ERR_SHAPE);
            const int p = kc->layer_pool[layer];
            const int ring = kind == HMD_SWA && x->window >= 1
                                 ? (x->window + kc->page_tokens - 1) / kc->page_tokens
                                 : 0;
            st = attn_run(static_cast<hmd_kind_t>(kind), x->window, ring, 1, x->B, x->H, x->Hkv,
                          x->d, kc->page_tokens, x->q, x->k, x->v, kc->k_pools[p], kc->v_pools[p],
                          kc->n_pages, x->page_table, x->max_pages, x->seq_lens, x->max_seq_len,
                          x->o, workspace, ws_bytes, rows + off[kind], n, stream);
        }
        if (st != HMD_OK) return st;
    }
    return HMD_OK;
}

}  // extern "C"

// attn_decode_static_ws: attn_decode for callers that cannot allocate device memory.
//
// attn_decode needs a caller-provided workspace for its split-K partials. Some callers have no
// way to obtain one: a plugin whose host application owns every byte of device memory through
// its own allocator and exposes none of it, or a serving loop that forbids device allocation
// after start-up so that its latency and memory footprint stay fixed. This entry point takes the
// same inputs and outputs as attn_decode but draws its workspace from a fixed array compiled
// into the library, so it calls no allocator at all.
//
// The array below is a file-scope __device__ variable of kStaticWsBytes bytes. Every GPU on
// which the library is loaded holds one copy of it until the process exits. In host code its
// name does not denote a device address, so its address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and cached; the first call on each device
// performs this set-up. Every call shares the same array and leaves its contents behind. Nothing
// in it needs clearing between calls, because each launch writes every partial it later reads.
// Calls whose work overlaps on the GPU (on different streams, or on different host threads
// without ordering) race on the array and must not be issued.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/hmd.h"
#include "kernels.h"

namespace {

constexpr size_t kStaticWsBytes = 16u << 20;  // 16 MiB
constexpr int kMaxDevices = hmd::kMaxDevices;

__device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

std::mutex g_mu;
void *g_ws_ptr[kMaxDevices] = {};

// Device address of g_static_ws on the current device (looked up once per device).
hmd_status_t static_ws_ptr(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return HMD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ws_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) {
            cudaGetLastError();
            return HMD_ERR_CUDA;
        }
        g_ws_ptr[dev] = p;
    }
    *out = g_ws_ptr[dev];
    return HMD_OK;
}

}  // namespace

extern "C" {

hmd_status_t attn_decode_static_ws(hmd_kind_t kind, int window, int B, int Hq, int Hkv, int d,
                                   int page_tokens, const void *q, const void *new_k,
                                   const void *new_v, void *k_pool, void *v_pool, int n_pages,
                                   const int32_t *page_table, int max_pages,
                                   const int32_t *seq_lens, int max_seq_len, void *o,
                                   hmd_stream_t stream) {
    if (B > 0 && Hq > 0 && Hkv > 0 && d > 0 && max_seq_len > 0) {
        const size_t need = attn_decode_workspace_size(kind, window, B, Hq, Hkv, d, page_tokens,
                                                       max_seq_len);
        if (need > kStaticWsBytes)  // too large for the fixed array
            return hmd::record_status(HMD_ERR_UNSUPPORTED);
    }
    void *ws = nullptr;
    const hmd_status_t st = static_ws_ptr(&ws);
    if (st != HMD_OK) return hmd::record_status(st);
    return attn_decode(kind, window, B, Hq, Hkv, d, page_tokens, q, new_k, new_v, k_pool, v_pool,
                       n_pages, page_table, max_pages, seq_lens, max_seq_len, o, ws,
                       kStaticWsBytes, stream);
}

}  // extern "C"

// Host-side construction of TMA tensor maps (cuTensorMapEncodeTiled, looked up through the
// runtime's driver entry point so the library does not link libcuda directly).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"

namespace hmd {

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode() {
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
}  // namespace

// A 2-D row-major tensor [rows][cols] read and written in boxes of [box_rows][box_cols], no
// swizzle; elements outside the tensor read as zero and are not written.
bool make_tmap_2d(CUtensorMap *m, CUtensorMapDataType dt, int esize, void *base, long long cols,
                  long long rows, int box_cols, int box_rows) {
    EncodeTiledFn enc = encode();
    if (!enc) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)cols * esize};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, dt, 2, base, gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The K or V input of a prompt, [n_tok][heads][d] bf16 (n_tok = B*T), as a 3-D tensor
// (d, heads, n_tok) read in boxes of (64 dims, 1 head, 64 tokens) with the 128-byte swizzle:
// one box is a [64 tokens][128 B] tile. Tokens past n_tok read as zero.
bool make_tmap_tokens_sw128(CUtensorMap *m, void *base, long long n_tok, int heads, int d) {
    EncodeTiledFn enc = encode();
    if (!enc) return false;
    const cuuint64_t gdim[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)n_tok};
    const cuuint64_t gstride[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, gdim, gstride, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// A [B][T][H][d] activation (bf16 or fp32) as a 4-D tensor (d, H, T, B) read in boxes of
// (box_d channels, 1 head, 64 tokens, 1 sequence): one box is a [64 tokens][box_d] tile,
// 128-byte swizzled if sw128. Tokens past T read as zero, so a chunk never reaches into the
// next sequence.
bool make_tmap_bthd(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, int B,
                    int T, int H, int d, int box_d, bool sw128) {
    EncodeTiledFn enc = encode();
    if (!enc) return false;
    const cuuint64_t gdim[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t gstride[3] = {(cuuint64_t)d * esize, (cuuint64_t)H * d * esize,
                                   (cuuint64_t)T * H * d * esize};
    const cuuint32_t box[4] = {(cuuint32_t)box_d, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, dt, 4, const_cast<void *>(base), gdim, gstride, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE,
               sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// A paged pool [n_pages][heads][64][d] bf16 viewed as [n_pages*heads*64 rows][d], read in boxes
// of 64 rows x 64 dims with the 128-byte swizzle: one box is half of one page of one head.
bool make_tmap_pool_sw128(CUtensorMap *m, void *pool, int n_pages, int heads, int d) {
    EncodeTiledFn enc = encode();
    if (!enc) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)d, (cuuint64_t)n_pages * heads * 64};
    const cuuint64_t gstride[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64, 64};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pool, gdim, gstride, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

}  // namespace hmd

// TMA descriptors (cuTensorMapEncodeTiled, reached through the runtime's driver entry point so the
// library does not link libcuda directly).
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace slra {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        else
            cudaGetLastError();
    });
    return fn;
}

}  // namespace

// 2D fp16 map over a head-major [rows][D] buffer: box 64 columns x box_rows rows, 128-B swizzle.
bool make_map_headmajor(CUtensorMap* m, const void* base, uint64_t rows, int D, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4D bf16 map over a [B][L][Hh][D] input with element strides st (D contiguous; token-major when
// contiguous): coordinates (d, head, token, batch), box 64 x 1 x box_tokens x 1, 128-B swizzle; tokens
// past L read as zero.
bool make_map_tokens(CUtensorMap* m, const void* base, int B, int L, int Hh, int D, const Strides& st,
                     int box_tokens) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hh), static_cast<cuuint64_t>(L),
                          static_cast<cuuint64_t>(B)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(st.h) * 2, static_cast<cuuint64_t>(st.l) * 2,
                             static_cast<cuuint64_t>(st.b) * 2};
    cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_tokens), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4D map over the output [B][L][Hh][D] (element strides st, D contiguous) for 64-token TMA stores of
// 128-byte column boxes (32 fp32 or 64 bf16 columns), 128-B swizzle on the shared-memory side; tokens
// past L are not written.
bool make_map_out(CUtensorMap* m, void* base, int B, int L, int Hh, int D, const Strides& st, bool f32) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t es = f32 ? 4 : 2;
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hh), static_cast<cuuint64_t>(L),
                          static_cast<cuuint64_t>(B)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(st.h) * es, static_cast<cuuint64_t>(st.l) * es,
                             static_cast<cuuint64_t>(st.b) * es};
    cuuint32_t box[4] = {f32 ? 32u : 64u, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Split count of the low-rank partial sums.  head_dim 128 (tensor-core kernel): ranges of 128-token
// tiles sized so a persistent grid of 148 CTAs gets about eight work items each; otherwise (CUDA-core
// kernel, 32-token steps) about two CTAs per SM.
int lowrank_nsplit(const Geom& g) {
    if (g.D == 128) {
        const long long ntiles = (g.L + 127) / 128;
        long long tps = static_cast<long long>(g.BH()) * ntiles / (148 * 8);
        tps = tps < 1 ? 1 : (tps > 64 ? 64 : tps);
        return static_cast<int>((ntiles + tps - 1) / tps);
    }
    const long long ntiles = (g.L + 31) / 32;
    long long ns = (2 * 148 + g.BH() - 1) / g.BH();
    ns = ns < 1 ? 1 : (ns > ntiles ? ntiles : ns);
    return static_cast<int>(ns);
}

}  // namespace slra

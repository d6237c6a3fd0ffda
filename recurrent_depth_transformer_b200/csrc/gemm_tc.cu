// Single-CTA instantiations of the tcgen05 GEMM (bf16 and tf32, every epilogue), the
// dispatcher, and the tensor-map encoder. The kernel itself is in gemm_tc.cuh.
#include "gemm_tc.cuh"

namespace rdt {

namespace {

template <typename T, int BN>
rdt_status dispatch_router(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap* tA2,
                           const CUtensorMap* tB2, const GemmArgs& args, const EpiParams& epi,
                           cudaStream_t st) {
    return launch<T, BN, EPI_TOPK, 1>(tA, tB, tA2, tB2, args, epi, st);
}

}  // namespace

rdt_status gemm_tc(bool bf16_elems, int bn, const CUtensorMap& tA, const CUtensorMap& tB,
                   const CUtensorMap* tA2, const CUtensorMap* tB2, const GemmArgs& args,
                   const EpiParams& epi, cudaStream_t st) {
    // a K split leaves partial sums to combine: only epilogues that reduce into their output
    // (and the router's, which combines its partial logits itself) may split
    if (args.split_k > 1 && epi.kind != EPI_SCATTER && epi.kind != EPI_OPROJ_LOOP && epi.kind != EPI_TOPK) {
        set_error("gemm_tc: a K split needs an epilogue that reduces into its output");
        return RDT_ERR_INVALID_ARG;
    }
    if (args.split_k > 1 && epi.kind == EPI_OPROJ_LOOP && epi.h_in) {
        set_error("gemm_tc: the O projection's stores of y and h_next need the whole K");
        return RDT_ERR_INVALID_ARG;
    }
    if (epi.kind == EPI_TOPK) {
        if (bf16_elems) {
            if (bn == 64) return dispatch_router<bf16, 64>(tA, tB, tA2, tB2, args, epi, st);
            if (bn == 128) return dispatch_router<bf16, 128>(tA, tB, tA2, tB2, args, epi, st);
            if (bn == 256) return dispatch_router<bf16, 256>(tA, tB, tA2, tB2, args, epi, st);
        } else {
            if (bn == 64) return dispatch_router<float, 64>(tA, tB, tA2, tB2, args, epi, st);
        }
        set_error("router: unsupported expert count");
        return RDT_ERR_UNSUPPORTED;
    }
    if (args.pair) {
        if (!bf16_elems) {
            set_error("gemm_tc: pair tiles need bf16 operands");
            return RDT_ERR_UNSUPPORTED;
        }
        return gemm_tc_pair(bn, tA, tB, tA2, tB2, args, epi, st);
    }
    if (bf16_elems) {
        if (bn == 128) return dispatch_kind<bf16, 128, 1>(tA, tB, tA2, tB2, args, epi, st);
        if (bn == 160) return dispatch_kind<bf16, 160, 1>(tA, tB, tA2, tB2, args, epi, st);
        if (bn == 256) return dispatch_kind<bf16, 256, 1>(tA, tB, tA2, tB2, args, epi, st);
    } else {
        if (bn == 128) return dispatch_kind<float, 128, 1>(tA, tB, tA2, tB2, args, epi, st);
    }
    set_error("gemm_tc: unsupported tile width");
    return RDT_ERR_UNSUPPORTED;
}

int num_sms() {
    static int n[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!n[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 148;
    }
    return n[dev];
}

// ----------------------------------------------------------------------------- tensor maps

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}
}  // namespace

rdt_status make_tmap_2d(CUtensorMap* map, const void* base, bool bf16_elems, uint64_t inner,
                        uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                        uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        set_error("cuTensorMapEncodeTiled entry point unavailable");
        return RDT_ERR_CUDA;
    }
    if ((reinterpret_cast<uintptr_t>(base) & 15) || (row_stride_bytes & 15)) {
        set_error("tensor map: base or row stride not 16-byte aligned");
        return RDT_ERR_MISALIGNED;
    }
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, bf16_elems ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                    2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed with code " + std::to_string(static_cast<int>(r)));
        return RDT_ERR_CUDA;
    }
    return RDT_OK;
}

}  // namespace rdt

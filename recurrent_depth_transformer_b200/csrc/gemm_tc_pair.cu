// CTA-pair instantiations of the tcgen05 GEMM (cta_group::2, 256-row tiles, bf16 operands,
// BN = 128, 192 or 256, every epilogue but the router's). The kernel is in gemm_tc.cuh.
#include "gemm_tc.cuh"

namespace rdt {

rdt_status gemm_tc_pair(int bn, const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap* tA2,
                        const CUtensorMap* tB2, const GemmArgs& args, const EpiParams& epi,
                        cudaStream_t st) {
    if (epi.kind == EPI_TOPK) {
        set_error("gemm_tc: the router runs on single-CTA tiles");
        return RDT_ERR_UNSUPPORTED;
    }
    if (bn == 128) return dispatch_kind<bf16, 128, 2>(tA, tB, tA2, tB2, args, epi, st);
    if (bn == 192) return dispatch_kind<bf16, 192, 2>(tA, tB, tA2, tB2, args, epi, st);
    if (bn == 256) return dispatch_kind<bf16, 256, 2>(tA, tB, tA2, tB2, args, epi, st);
    set_error("gemm_tc: unsupported pair tile width");
    return RDT_ERR_UNSUPPORTED;
}

}  // namespace rdt

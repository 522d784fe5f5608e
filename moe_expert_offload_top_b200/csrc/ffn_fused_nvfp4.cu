// Fused decode FFN (ffn_fused.cuh) for NVFP4 expert weights; one source per weight
// format so the instantiations compile in parallel.
#include "ffn_fused.cuh"

namespace ftk {

cudaError_t launch_ffn_fused_nvfp4(int nt, int rg, int rd, const FusedParams& p, const ExpertList& list, int num_sms,
                              cudaStream_t s) {
  return fused::launch_wt<gemv::WT_NVFP4>(nt, rg, rd, p, list, num_sms, s);
}

}  // namespace ftk

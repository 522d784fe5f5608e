// Fused decode FFN (ffn_fused.cuh) for fp32 expert weights; one source per weight
// format so the instantiations compile in parallel.
#include "ffn_fused.cuh"

namespace ftk {

cudaError_t launch_ffn_fused_f32(int nt, int rg, int rd, const FusedParams& p, const ExpertList& list, int num_sms,
                              cudaStream_t s) {
  return fused::launch_wt<gemv::WT_F32>(nt, rg, rd, p, list, num_sms, s);
}

}  // namespace ftk

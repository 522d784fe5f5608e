// Decode expert FFN + combine with its scratch in a static device array, for
// callers that may not allocate device memory.
//
// The intermediate SwiGLU activations h [(T*k + T) x I] and the expert outputs
// y [(T*k + T) x H] (fp32) live in g_ffn_scratch, a file-scope array of
// kNoAllocFloats floats that every GPU which loads this library holds until the
// process exits.  Host code never passes the array's name to a kernel: the
// array's device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and cached.
#include <mutex>
#include <string>

#include "../../include/ftmoe.h"
#include "kernels.hpp"

namespace {

constexpr size_t kNoAllocFloats = FT_NOALLOC_SCRATCH_FLOATS;
static __device__ __align__(256) float g_ffn_scratch[kNoAllocFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_addr[kMaxDevices] = {};

// Device address of g_ffn_scratch on the current device (looked up on first use).
cudaError_t scratch_for_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_ffn_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

namespace ftk {
void set_step_error(const std::string& msg);
}

extern "C" int ft_expert_ffn_decode_noalloc(const void* x, int T, int H, int I, int top_k, int wdtype,
                                            const void* const* blobs, const int* experts, int n_list,
                                            int max_pairs_per_expert, const int* offsets, const int* perm,
                                            const float* gates, const int* inv, int has_shared, void* out,
                                            void* stream) {
  if (T < 0 || H < 8 || I < 8 || H % 8 || I % 8 || top_k < 1 || n_list < 0 ||
      n_list > ftk::kMaxList || wdtype < FT_W_F32 || wdtype > FT_W_NVFP4 ||
      (wdtype == FT_W_INT4_G128 && (H % 128 || I % 128)) || (wdtype == FT_W_NVFP4 && (H % 32 || I % 32)) ||
      (T > 0 && (!x || !offsets || !perm || !gates || !inv || !out)) ||
      (n_list > 0 && (!blobs || !experts))) {
    ftk::set_step_error("ft_expert_ffn_decode_noalloc: invalid argument");
    return FT_ERR_INVALID;
  }
  const unsigned long long rows = (unsigned long long)T * top_k + (unsigned long long)T;
  const unsigned long long need = rows * ((unsigned long long)I + (unsigned long long)H);
  if (need > kNoAllocFloats) {
    ftk::set_step_error("ft_expert_ffn_decode_noalloc: (T*k + T) * (I + H) = " + std::to_string(need) +
                        " floats exceeds the static scratch of " + std::to_string(kNoAllocFloats) +
                        " floats (FT_NOALLOC_SCRATCH_FLOATS)");
    return FT_ERR_INVALID;
  }
  if (T == 0) return FT_OK;
  ftk::ExpertList list;
  list.n = n_list;
  int n_shared = 0;
  for (int i = 0; i < n_list; ++i) {
    if (experts[i] < -1 || experts[i] >= FT_MAX_EXPERTS || !blobs[i]) {
      ftk::set_step_error("ft_expert_ffn_decode_noalloc: bad expert list entry");
      return FT_ERR_INVALID;
    }
    n_shared += experts[i] < 0;
    list.expert[i] = experts[i];
    list.blob[i] = static_cast<const uint8_t*>(blobs[i]);
  }
  // the combine reads the shared expert's rows exactly when has_shared is set: they must be
  // written by this call, not left in the shared array by an earlier one
  if ((has_shared != 0) != (n_shared == 1) || n_shared > 1) {
    ftk::set_step_error("ft_expert_ffn_decode_noalloc: has_shared needs exactly one list entry -1, "
                        "and no such entry without it");
    return FT_ERR_INVALID;
  }
  float* scratch = nullptr;
  cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) {
    ftk::set_step_error(std::string("ft_expert_ffn_decode_noalloc: cudaGetSymbolAddress: ") +
                        cudaGetErrorString(e));
    return FT_ERR_CUDA;
  }
  float* h = scratch;
  float* y = scratch + rows * (unsigned long long)I;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  e = ftk::launch_ffn_decode(x, T, H, I, top_k, wdtype, list, max_pairs_per_expert, offsets, perm, h, y, s,
                             nullptr);
  if (e == cudaSuccess)
    e = ftk::launch_combine(y, gates, inv, T, H, top_k, has_shared != 0, wdtype != FT_W_F32, out, s);
  if (e != cudaSuccess) {
    ftk::set_step_error(std::string("ft_expert_ffn_decode_noalloc: launch: ") + cudaGetErrorString(e));
    return FT_ERR_CUDA;
  }
  return FT_OK;
}

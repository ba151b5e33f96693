// topk.cu -- the top-k selection in 512-thread CTAs (two per SM), and the
// choice between the two widths the selection is built at.
#define DSA_TOPK_THREADS 512
#define DSA_TOPK_MIN_CTAS 2
#define DSA_TOPK_LAUNCH launch_topk_wide
#include "topk_impl.cuh"

namespace dsa {

cudaError_t launch_topk_narrow(const TopkArgs& a, cudaStream_t st);

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st) {
  return a.narrow ? launch_topk_narrow(a, st) : launch_topk_wide(a, st);
}

}  // namespace dsa

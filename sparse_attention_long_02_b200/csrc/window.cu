// window.cu -- index sets for sliding-window and dense causal attention.
//
// Sliding-window attention lets a token attend only to a fixed number of the
// keys just before it ("m.gxzdkb.com/media/457.html", section "秘密武器";
// "oilbeater.com ... deepseek-sparse-attention", section "Sparse Attention"),
// and DSA generalises it by choosing the keys with the indexer instead of by
// distance. Writing the window as an index set lets the sparse MLA kernel run
// it unchanged; a window that covers the whole causal prefix gives dense
// causal attention, the full interface the pages keep beside DSA
// ("ele-yufo.com/posts/deepseek-v3-2-exp", section "六、实测表现与取舍").
//
// Row t (position p = q_pos0 + t, clamped to the last key S-1) selects keys
// max(0, p - window + 1) .. p in increasing order, then -1 up to k.
#include "dsa_internal.h"

namespace dsa {
namespace {

__global__ void __launch_bounds__(256) window_kernel(int T, int S, int q_pos0, int window, int k,
                                                     int* __restrict__ idx) {
  const int t = blockIdx.x;
  if (t >= T) return;
  const long long p = min(static_cast<long long>(q_pos0) + t, static_cast<long long>(S) - 1);
  const long long lo = max(0ll, p - window + 1);
  const long long n = p - lo + 1;                 // <= window <= k
  int4* row = reinterpret_cast<int4*>(idx + static_cast<long long>(t) * k);
  for (int j4 = threadIdx.x; j4 < k / 4; j4 += blockDim.x) {
    int v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const long long j = 4ll * j4 + e;
      v[e] = j < n ? static_cast<int>(lo + j) : -1;
    }
    row[j4] = make_int4(v[0], v[1], v[2], v[3]);
  }
}

}  // namespace

cudaError_t launch_window(int T, int S, int q_pos0, int window, int k, int* idx, cudaStream_t st) {
  window_kernel<<<T, 256, 0, st>>>(T, S, q_pos0, window, k, idx);
  return cudaGetLastError();
}

}  // namespace dsa

// decode_static.cu -- paged decode for callers that cannot allocate device
// memory.
//
// dsa_decode_paged() takes its scratch (the per-query score rows and the
// selected indices) from a workspace the caller allocates. Some callers
// cannot do that: code that runs where cudaMalloc is forbidden or unsafe,
// such as a host callback or a plugin inside another framework's allocator,
// or a caller with no device allocator at all. dsa_decode_paged_noalloc()
// serves them with a scratch area that is a fixed, file-scope device array:
// it is part of the library's image, so every GPU that loads the library
// holds it until the process exits, and no call allocates anything.
//
// The array's host-side name is only a stand-in for the device object, so
// the host looks up its device address once per device (with that device
// current) through cudaGetSymbolAddress and passes that address on. The
// work itself is done by dsa_decode_paged(), with this array as its
// workspace.
#include <mutex>

#include "../../include/dsa.h"
#include "dsa_internal.h"

namespace {

// Largest scratch a call may need, see dsa_decode_paged_workspace_size().
constexpr size_t kScratchBytes = size_t(32) << 20;   // 32 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, looked up on
// the first call made with that device current.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    dsa::set_last_error("dsa_decode_paged_noalloc: no usable current device");
    return DSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      dsa::set_last_error("dsa_decode_paged_noalloc: cudaGetSymbolAddress of the scratch failed");
      return DSA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return DSA_OK;
}

}  // namespace

extern "C" int dsa_decode_paged_noalloc(
    const void* q8, const float* q_scale, const float* w, const void* q, const void* k8_pool,
    const float* k_scale_pool, const void* kv_pool, const int32_t* block_table,
    const int32_t* seq_len, int B, int nq, int max_blocks, int nblk, int Hi, int H, int k,
    float scale, float sm_scale, int32_t* idx_out, void* out, float* lse, dsa_stream_t stream) {
  if (B < 0 || nq < 1 || max_blocks < 1 || k <= 0) return DSA_ERR_INVALID_ARG;
  if (B == 0) return DSA_OK;
  const size_t need = dsa_decode_paged_workspace_size(B, nq, max_blocks, Hi, H, k);
  if (need == 0) return DSA_ERR_INVALID_ARG;
  if (need > kScratchBytes) {
    dsa::set_last_error(
        "dsa_decode_paged_noalloc: B*nq*(64*max_blocks*4 + 4*k) bytes exceed the 32 MiB static "
        "scratch; use dsa_decode_paged with a caller workspace");
    return DSA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  const int s = scratch_address(&scratch);
  if (s != DSA_OK) return s;
  return dsa_decode_paged(q8, q_scale, w, q, k8_pool, k_scale_pool, kv_pool, block_table, seq_len,
                          B, nq, max_blocks, nblk, Hi, H, k, scale, sm_scale, idx_out, out, lse,
                          scratch, kScratchBytes, stream);
}

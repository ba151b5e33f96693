// api.cu -- the C ABI of libdsa.so (declared in include/dsa.h): host-side
// argument checks, tensor-map construction, workspace carving and the launch
// sequence of each entry point. No device memory is allocated here.
#include <cstdio>
#include <mutex>

#include "../../include/dsa.h"
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {

// Per-device status words, [0] the error bits and [1] the debug bits;
// kernels get the address of [0] as an argument.
__device__ unsigned g_error_word[2];

namespace {

constexpr int kMaxDevices = 64;
unsigned* g_err_ptr[kMaxDevices] = {};
std::mutex g_mu;

// Address of the current device's error word (looked up once per device).
unsigned* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<unsigned*>(p);
  }
  return g_err_ptr[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// The tcgen05 GEMM tiles its M rows 128 to a CTA along grid.y (at most 65535).
constexpr long long kMaxGemmRows = 65535ll * 128;

thread_local char g_last_error[256] = "";

int status_of(cudaError_t e) {
  if (e == cudaSuccess) return DSA_OK;
  snprintf(g_last_error, sizeof g_last_error, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return DSA_ERR_CUDA;
}

}  // namespace

void set_last_error(const char* msg) { snprintf(g_last_error, sizeof g_last_error, "%s", msg); }

cudaError_t make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         uint64_t inner, uint64_t rows, uint64_t row_stride, uint32_t box_inner,
                         uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_stride};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace dsa

using namespace dsa;

namespace {

bool valid_hi(int Hi) {
  return Hi == 1 || Hi == 2 || Hi == 4 || Hi == 8 || Hi == 16 || Hi == 32 || Hi == 64;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Per-device stream and events that let the top-k of one prefill chunk run
// beside the indexer of the next (created once, no device memory). Calls on
// one device enqueue under a lock so the events are recorded and waited on in
// order.
struct Overlap {
  cudaStream_t side = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t idx_done[2] = {nullptr, nullptr};
  cudaEvent_t topk_done[2] = {nullptr, nullptr};
  bool ready = false;
};
constexpr int kMaxDev = 64;
Overlap g_overlap[kMaxDev];
std::mutex g_overlap_mu;

Overlap* overlap_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  Overlap& o = g_overlap[dev];
  if (!o.ready) {
    bool ok = cudaStreamCreateWithFlags(&o.side, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&o.start, cudaEventDisableTiming) == cudaSuccess;
    for (int b = 0; ok && b < 2; ++b)
      ok = cudaEventCreateWithFlags(&o.idx_done[b], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&o.topk_done[b], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return nullptr;
    o.ready = true;
  }
  return &o;
}

int run_indexer(const void* q8, const float* q_scale, const void* k8, const float* k_scale,
                const float* w, int T, int S, int Hi, int q_pos0, float scale, float* scores,
                int64_t ld, cudaStream_t st) {
  IndexerArgs a;
  a.T = T;
  a.S = S;
  a.Hi = Hi;
  a.q_pos0 = q_pos0;
  a.scale = scale;
  a.w = w;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.scores = scores;
  a.ld = ld;
  a.err = device_error_word();
  if (!a.err) return DSA_ERR_CUDA;
  return status_of(launch_indexer(a, q8, k8, S, st));
}

int run_topk(const float* scores, int rows, int S, int64_t ld, int q_pos0, const int* seq_len,
             int nq, int k, int32_t* idx, cudaStream_t st, bool narrow = false) {
  TopkArgs a;
  a.narrow = narrow;
  a.scores = scores;
  a.ld = ld;
  a.rows = rows;
  a.k = k;
  a.q_pos0 = q_pos0;
  a.S = S;
  a.seq_len = seq_len;
  a.nq = nq;
  a.idx = idx;
  a.err = device_error_word();
  if (!a.err) return DSA_ERR_CUDA;
  return status_of(launch_topk(a, st));
}

}  // namespace

extern "C" {

const char* dsa_status_string(int status) {
  switch (status) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case DSA_ERR_WORKSPACE: return "workspace missing or too small";
    case DSA_ERR_CUDA: return "CUDA runtime error";
    case DSA_ERR_TIMEOUT: return "kernel wait timed out";
    case DSA_ERR_DEVICE_BOUNDS: return "kernel met an out-of-range index";
    case DSA_ERR_NOT_IMPLEMENTED: return "not implemented";
    default: return "unknown status";
  }
}

int dsa_version(void) { return 100; }

const char* dsa_last_error_string(void) { return g_last_error; }

int dsa_get_device_error(dsa_stream_t stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  unsigned* p = device_error_word();
  if (!p) return DSA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (v != 0 && cudaMemset(p, 0, sizeof v) != cudaSuccess) return DSA_ERR_CUDA;
  if (v & kErrTimeout) return DSA_ERR_TIMEOUT;
  if (v & kErrBounds) return DSA_ERR_DEVICE_BOUNDS;
  return DSA_OK;
}

int dsa_debug_stall(unsigned mask) {
  if (mask & ~static_cast<unsigned>(DSA_DEBUG_STALL_INDEXER | DSA_DEBUG_STALL_MLA))
    return DSA_ERR_INVALID_ARG;
  unsigned* p = device_error_word();
  if (!p) return DSA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return DSA_ERR_CUDA;
  return status_of(cudaMemcpy(p + 1, &mask, sizeof mask, cudaMemcpyHostToDevice));
}

int dsa_indexer_scores(const void* q8, const float* q_scale, const void* k8, const float* k_scale,
                       const float* w, int T, int S, int Hi, int q_pos0, float scale,
                       float* scores, int64_t ld, dsa_stream_t stream) {
  if (!q8 || !k8 || !w || !scores || T < 0 || S < 0 || q_pos0 < 0 || !(scale > 0.f) ||
      ld < S || (ld & 3) || !aligned16(q8) || !aligned16(k8) || !aligned16(scores))
    return DSA_ERR_INVALID_ARG;
  if (!valid_hi(Hi)) return DSA_ERR_UNSUPPORTED;
  if (T == 0 || S == 0) return DSA_OK;
  return run_indexer(q8, q_scale, k8, k_scale, w, T, S, Hi, q_pos0, scale, scores, ld,
                     static_cast<cudaStream_t>(stream));
}

int dsa_topk(const float* scores, int T, int S, int64_t ld, int q_pos0, int k, int32_t* idx,
             dsa_stream_t stream) {
  if (!scores || !idx || T < 0 || S < 0 || q_pos0 < 0 || k <= 0 || k > 65536 || (k & 3) ||
      ld < S || (ld & 3) || !aligned16(scores) || !aligned16(idx))
    return DSA_ERR_INVALID_ARG;
  if (T == 0) return DSA_OK;
  return run_topk(scores, T, S, ld, q_pos0, nullptr, 1, k, idx, static_cast<cudaStream_t>(stream));
}

size_t dsa_project_workspace_size(int T, int Hi) {
  if (T <= 0 || !valid_hi(Hi)) return 0;
  return round_up(static_cast<size_t>(T) * (Hi * 128 + 128) * 4, 256) +
         2 * round_up(static_cast<size_t>(T) * 4, 256);
}

int dsa_project_indexer_inputs(const void* h, const void* wt, const float* rope, int T, int d,
                               int Hi, void* q8, float* q_scale, void* k8, float* k_scale, float* a,
                               void* workspace, size_t ws_bytes, dsa_stream_t stream) {
  if (!h || !wt || !rope || !q8 || !q_scale || !k8 || !k_scale || !a || T < 0 || d < 8 ||
      (d & 7) || T > kMaxGemmRows || !aligned16(h) || !aligned16(wt) || !aligned16(rope) ||
      !aligned16(q8) || !aligned16(k8) || !aligned16(a))
    return DSA_ERR_INVALID_ARG;
  if (!valid_hi(Hi)) return DSA_ERR_UNSUPPORTED;
  if (T == 0) return DSA_OK;
  const size_t need = dsa_project_workspace_size(T, Hi);
  if (!workspace || !aligned16(workspace) || ws_bytes < need) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProjArgs P;
  P.T = T;
  P.d = d;
  P.Hi = Hi;
  P.N = Hi * 128 + 128 + Hi;
  P.rope = rope;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  P.y = reinterpret_cast<float*>(ws);
  const size_t ybytes = round_up(static_cast<size_t>(T) * (Hi * 128 + 128) * 4, 256);
  P.amax_q = reinterpret_cast<unsigned*>(ws + ybytes);
  P.amax_k = reinterpret_cast<unsigned*>(ws + ybytes + round_up(static_cast<size_t>(T) * 4, 256));
  P.a = a;
  P.q8 = static_cast<uint8_t*>(q8);
  P.k8 = static_cast<uint8_t*>(k8);
  P.q_scale = q_scale;
  P.k_scale = k_scale;
  P.err = device_error_word();
  cudaError_t e = cudaMemsetAsync(ws + ybytes, 0, 2 * round_up(static_cast<size_t>(T) * 4, 256), st);
  if (e == cudaSuccess) e = launch_project(P, h, wt, st);
  return status_of(e);
}

size_t dsa_attention_probs_workspace_size(int T, int S, int H) {
  if (T <= 0 || S <= 0 || H < 1) return 0;
  return static_cast<size_t>(T) * H * round_up(static_cast<size_t>(S), 4) * 4;
}

int dsa_attention_probs_mean(const void* q, const void* kv, const float* lse, int T, int S,
                             int H, int q_pos0, float sm_scale, float* p, int64_t ldp,
                             void* workspace, size_t ws_bytes, dsa_stream_t stream) {
  if (!q || !kv || !lse || !p || T < 0 || S <= 0 || q_pos0 < 0 || H < 1 || H > 128 ||
      ldp < S || !(sm_scale > 0.f) || !aligned16(q) || !aligned16(kv) ||
      static_cast<long long>(T) * H > kMaxGemmRows)
    return DSA_ERR_INVALID_ARG;
  if (T == 0) return DSA_OK;
  const size_t need = dsa_attention_probs_workspace_size(T, S, H);
  if (!workspace || !aligned16(workspace) || ws_bytes < need) return DSA_ERR_WORKSPACE;
  return status_of(launch_attention_probs(q, kv, lse, T, S, H, q_pos0, sm_scale, p, ldp,
                                          static_cast<float*>(workspace),
                                          static_cast<long long>(round_up(S, 4)),
                                          device_error_word(), static_cast<cudaStream_t>(stream)));
}

int dsa_indexer_kl(const float* I, int64_t ldi, const float* p, int64_t ldp, int T, int S,
                   int q_pos0, float* loss, float* grad, int64_t ldg, dsa_stream_t stream) {
  if (!I || !p || !loss || !grad || T < 0 || S <= 0 || q_pos0 < 0 || ldi < S || ldp < S ||
      ldg < S)
    return DSA_ERR_INVALID_ARG;
  if (T == 0) return DSA_OK;
  return status_of(launch_indexer_kl(I, ldi, p, ldp, T, S, q_pos0, loss, grad, ldg,
                                     static_cast<cudaStream_t>(stream)));
}

size_t dsa_indexer_backward_workspace_size(int T, int S, int Hi) {
  if (T <= 0 || S <= 0 || !valid_hi(Hi)) return 0;
  return dsa::indexer_backward_workspace(T, S, Hi);
}

int dsa_indexer_backward(const void* q8, const float* q_scale, const void* k8, const float* k_scale,
                         const float* w, int T, int S, int Hi, int q_pos0, float scale,
                         const float* grad, int64_t ldg, float* dq, float* dk, float* dw,
                         void* workspace, size_t ws_bytes, dsa_stream_t stream) {
  if (!q8 || !k8 || !w || !grad || !dq || !dk || !dw || T < 0 || S <= 0 || q_pos0 < 0 ||
      ldg < S || !(scale > 0.f) || !aligned16(dq) || !aligned16(dk) ||
      S > kMaxGemmRows || static_cast<long long>(T) * Hi > kMaxGemmRows)
    return DSA_ERR_INVALID_ARG;
  if (!valid_hi(Hi)) return DSA_ERR_UNSUPPORTED;
  if (T == 0) return DSA_OK;
  if (!workspace || !aligned16(workspace) ||
      ws_bytes < dsa::indexer_backward_workspace(T, S, Hi))
    return DSA_ERR_WORKSPACE;
  IndexerBwdArgs a;
  a.T = T;
  a.S = S;
  a.Hi = Hi;
  a.q_pos0 = q_pos0;
  a.scale = scale;
  a.q8 = static_cast<const uint8_t*>(q8);
  a.q_scale = q_scale;
  a.k8 = static_cast<const uint8_t*>(k8);
  a.k_scale = k_scale;
  a.w = w;
  a.grad = grad;
  a.ldg = ldg;
  a.dq = dq;
  a.dk = dk;
  a.dw = dw;
  return status_of(launch_indexer_backward(a, workspace, device_error_word(),
                                           static_cast<cudaStream_t>(stream)));
}

int dsa_window_indices(int T, int S, int q_pos0, int window, int k, int32_t* idx,
                       dsa_stream_t stream) {
  if (!idx || T < 0 || S <= 0 || q_pos0 < 0 || window < 1 || k <= 0 || (k & 3) || window > k ||
      !aligned16(idx))
    return DSA_ERR_INVALID_ARG;
  if (T == 0) return DSA_OK;
  return status_of(dsa::launch_window(T, S, q_pos0, window, k, idx,
                                      static_cast<cudaStream_t>(stream)));
}

static int mla_common(const void* q, const void* kv, const int32_t* idx, int T, int S, int H, int k,
                      float sm_scale, void* out, float* lse, const int32_t* block_table,
                      const int32_t* seq_len, int max_blocks, int nblk, int nq,
                      cudaStream_t st, int dense = 0, int q_pos0 = 0, int compact = 0) {
  if (!q || !kv || (!idx && !dense) || !out || T < 0 || S < 0 || k <= 0 || (k & 3) ||
      !(sm_scale > 0.f) || q_pos0 < 0 || !aligned16(q) || !aligned16(kv) || !aligned16(idx) ||
      !aligned16(out))
    return DSA_ERR_INVALID_ARG;
  if (H < 1 || H > 128) return DSA_ERR_UNSUPPORTED;
  if (T == 0) return DSA_OK;
  MlaArgs a;
  a.T = T;
  a.S = S;
  a.H = H;
  a.k = k;
  a.sm_scale_log2 = sm_scale * 1.4426950408889634f;
  a.idx = idx;
  a.dense = dense;
  a.q_pos0 = q_pos0;
  a.compact = compact;
  a.block_table = block_table;
  a.seq_len = seq_len;
  a.max_blocks = max_blocks;
  a.nblk = nblk;
  a.nq = nq;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.err = device_error_word();
  if (!a.err) return DSA_ERR_CUDA;
  const long long kv_rows = block_table ? static_cast<long long>(nblk) * 64 : S;
  if (kv_rows <= 0) return DSA_ERR_INVALID_ARG;
  return status_of(launch_sparse_mla(a, q, kv, kv_rows, static_cast<long long>(T) * H, st));
}

int dsa_sparse_mla_fwd(const void* q, const void* kv, const int32_t* idx, int T, int S, int H,
                       int k, float sm_scale, void* out, float* lse, dsa_stream_t stream) {
  if (S <= 0 && T > 0) return DSA_ERR_INVALID_ARG;
  return mla_common(q, kv, idx, T, S, H, k, sm_scale, out, lse, nullptr, nullptr, 0, 0, 1,
                    static_cast<cudaStream_t>(stream));
}

int dsa_dense_causal_mla(const void* q, const void* kv, int T, int S, int H, int q_pos0,
                         float sm_scale, void* out, float* lse, dsa_stream_t stream) {
  if (S <= 0 && T > 0) return DSA_ERR_INVALID_ARG;
  return mla_common(q, kv, nullptr, T, S, H, 4, sm_scale, out, lse, nullptr, nullptr, 0, 0, 1,
                    static_cast<cudaStream_t>(stream), 1, q_pos0);
}

int dsa_dense_causal_mla_decode_paged(const void* q, const void* kv_pool,
                                      const int32_t* block_table, const int32_t* seq_len, int B,
                                      int nq, int max_blocks, int nblk, int H, float sm_scale,
                                      void* out, float* lse, dsa_stream_t stream) {
  if (!block_table || !seq_len || B < 0 || nq < 1 || max_blocks < 1 || nblk < 1)
    return DSA_ERR_INVALID_ARG;
  return mla_common(q, kv_pool, nullptr, B * nq, max_blocks * 64, H, 4, sm_scale, out, lse,
                    block_table, seq_len, max_blocks, nblk, nq, static_cast<cudaStream_t>(stream),
                    1, 0);
}

int dsa_sparse_mla_decode_paged(const void* q, const void* kv_pool, const int32_t* block_table,
                                const int32_t* seq_len, const int32_t* idx, int B, int nq,
                                int max_blocks, int nblk, int H, int k, float sm_scale, void* out,
                                float* lse, dsa_stream_t stream) {
  if (!block_table || !seq_len || B < 0 || nq < 1 || max_blocks < 1 || nblk < 1)
    return DSA_ERR_INVALID_ARG;
  return mla_common(q, kv_pool, idx, B * nq, max_blocks * 64, H, k, sm_scale, out, lse,
                    block_table, seq_len, max_blocks, nblk, nq, static_cast<cudaStream_t>(stream));
}

// The sparse MLA on a selection this library's top-k wrote: every row holds
// its selected slots first, so a row that sees fewer than k keys walks only
// those (rows of a contiguous cache at positions q_pos0 + r).
static int mla_own_selection(const void* q, const void* kv, const int32_t* idx, int T, int S,
                             int H, int k, int q_pos0, float sm_scale, void* out, float* lse,
                             cudaStream_t st) {
  if (S <= 0 && T > 0) return DSA_ERR_INVALID_ARG;
  return mla_common(q, kv, idx, T, S, H, k, sm_scale, out, lse, nullptr, nullptr, 0, 0, 1, st, 0,
                    q_pos0, 1);
}
static int mla_own_selection_paged(const void* q, const void* kv_pool, const int32_t* block_table,
                                   const int32_t* seq_len, const int32_t* idx, int B, int nq,
                                   int max_blocks, int nblk, int H, int k, float sm_scale,
                                   void* out, float* lse, cudaStream_t st) {
  return mla_common(q, kv_pool, idx, B * nq, max_blocks * 64, H, k, sm_scale, out, lse,
                    block_table, seq_len, max_blocks, nblk, nq, st, 0, 0, 1);
}

namespace {

// Sampled keys (the first 256 of every 4096) among keys 0 .. S-1.
long long sample_count(int S) {
  const long long p = S - 1;
  return (p >> 12) * 256 + std::min<long long>(p & 4095, 255) + 1;
}

// Workspace of the fused path, each part 256-byte aligned. The candidate
// lists and failure lists are double-buffered by chunk parity, so the
// selection of one chunk (side stream) overlaps the indexer passes of the
// next (caller's stream).
struct FusedLayout {
  long long M, ldm, ld;
  size_t k8s, kss, sample, tau, cnt[2], ckey[2], cidx[2], fail[2], fail_total, scratch, idx,
      total;
  int nbuf;
};

FusedLayout fused_layout(int T, int S, int k, int chunk) {
  FusedLayout L;
  const size_t rows = chunk <= 0 ? T : std::min(chunk, T);
  L.M = sample_count(S);
  L.ldm = static_cast<long long>(round_up(static_cast<size_t>(L.M), 4));
  L.ld = static_cast<long long>(round_up(static_cast<size_t>(S), 4));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, 256);
    return o;
  };
  L.k8s = take(static_cast<size_t>(L.M) * 128);
  L.kss = take(static_cast<size_t>(L.M) * 4);
  L.sample = take(rows * L.ldm * 4);
  L.tau = take(rows * 4);
  L.nbuf = rows < static_cast<size_t>(T) ? 2 : 1;
  for (int b = 0; b < 2; ++b) {
    const int u = b < L.nbuf ? b : 0;     // one chunk: both parities share a buffer
    if (u != b) {
      L.cnt[b] = L.cnt[0];
      L.ckey[b] = L.ckey[0];
      L.cidx[b] = L.cidx[0];
      L.fail[b] = L.fail[0];
      continue;
    }
    L.cnt[b] = take(rows * 4);
    L.ckey[b] = take(rows * kFusedCandCap * 4);
    L.cidx[b] = take(rows * kFusedCandCap * 4);
    L.fail[b] = take(4 + rows * 4);
  }
  L.fail_total = take(4);
  L.scratch = take(static_cast<size_t>(kFusedSlots) * L.ld * 4);
  L.idx = take(static_cast<size_t>(T) * k * 4);
  L.total = off;
  return L;
}

}  // namespace

size_t dsa_forward_workspace_size(int T, int S, int Hi, int H, int k, int chunk) {
  (void)Hi;
  (void)H;
  if (T <= 0 || S <= 0 || k <= 0) return 0;
  const size_t rows = chunk <= 0 ? T : std::min(chunk, T);
  const size_t ld = round_up(static_cast<size_t>(S), 4);
  const size_t nbuf = rows < static_cast<size_t>(T) ? 2 : 1;   // double-buffered chunks
  return nbuf * round_up(rows * ld * sizeof(float), 256) +
         round_up(static_cast<size_t>(T) * k * sizeof(int32_t), 256);
}

int dsa_forward(const void* q8, const float* q_scale, const void* k8, const float* k_scale,
                const float* w, const void* q, const void* kv, int T, int S, int Hi, int H,
                int q_pos0, int k, int chunk, float scale, float sm_scale, int32_t* idx_out,
                void* out, float* lse, void* workspace, size_t ws_bytes, dsa_stream_t stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!q8 || !k8 || !w || !q || !kv || !out || T < 0 || S < 0 || q_pos0 < 0 || k <= 0 ||
      k > 65536 || (k & 3) || !(scale > 0.f) || !(sm_scale > 0.f))
    return DSA_ERR_INVALID_ARG;
  if (!valid_hi(Hi)) return DSA_ERR_UNSUPPORTED;
  if (H < 1 || H > 128) return DSA_ERR_UNSUPPORTED;
  if (T == 0) return DSA_OK;
  if (S == 0) return DSA_ERR_INVALID_ARG;
  const size_t need = dsa_forward_workspace_size(T, S, Hi, H, k, chunk);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return DSA_ERR_WORKSPACE;
  const int rows = chunk <= 0 ? T : std::min(chunk, T);
  const int64_t ld = static_cast<int64_t>(round_up(static_cast<size_t>(S), 4));
  const size_t chunk_bytes = round_up(static_cast<size_t>(rows) * ld * 4, 256);
  const int nbuf = rows < T ? 2 : 1;
  float* scores[2] = {static_cast<float*>(workspace),
                      reinterpret_cast<float*>(static_cast<char*>(workspace) + chunk_bytes)};
  int32_t* idx = idx_out;
  if (!idx) idx = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + nbuf * chunk_bytes);
  if (!aligned16(idx)) return DSA_ERR_INVALID_ARG;
  const uint8_t* q8b = static_cast<const uint8_t*>(q8);
  auto indexer_chunk = [&](int c0, float* sc) {
    const int n = std::min(rows, T - c0);
    return dsa_indexer_scores(q8b + static_cast<size_t>(c0) * Hi * 128,
                              q_scale ? q_scale + c0 : nullptr, k8, k_scale,
                              w + static_cast<size_t>(c0) * Hi, n, S, Hi, q_pos0 + c0, scale, sc,
                              ld, stream);
  };
  // beside the next chunk's indexer, the selection runs in the narrow CTAs
  // that fit on an SM next to an indexer CTA
  auto topk_chunk = [&](int c0, float* sc, cudaStream_t on, bool beside) {
    const int n = std::min(rows, T - c0);
    return run_topk(sc, n, S, ld, q_pos0 + c0, nullptr, 1, k,
                    idx + static_cast<size_t>(c0) * k, on, beside);
  };
  std::unique_lock<std::mutex> lock(g_overlap_mu);
  Overlap* ov = nbuf == 2 ? overlap_for_current_device() : nullptr;
  if (!ov) {                               // one chunk (or no side stream): in order
    lock.unlock();
    for (int c0 = 0; c0 < T; c0 += rows) {
      int s = indexer_chunk(c0, scores[0]);
      if (s != DSA_OK) return s;
      s = topk_chunk(c0, scores[0], st, false);
      if (s != DSA_OK) return s;
    }
    return mla_own_selection(q, kv, idx, T, S, H, k, q_pos0, sm_scale, out, lse, st);
  }
  // top-k of chunk c (side stream) runs beside the indexer of chunk c+1
  cudaError_t e = cudaEventRecord(ov->start, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ov->side, ov->start, 0);
  if (e != cudaSuccess) return status_of(e);
  int c = 0;
  for (int c0 = 0; c0 < T; c0 += rows, ++c) {
    const int b = c & 1;
    if (c >= 2 && (e = cudaStreamWaitEvent(st, ov->topk_done[b], 0)) != cudaSuccess)
      return status_of(e);
    int s = indexer_chunk(c0, scores[b]);
    if (s != DSA_OK) return s;
    if ((e = cudaEventRecord(ov->idx_done[b], st)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(ov->side, ov->idx_done[b], 0)) != cudaSuccess)
      return status_of(e);
    s = topk_chunk(c0, scores[b], ov->side, true);
    if (s != DSA_OK) return s;
    if ((e = cudaEventRecord(ov->topk_done[b], ov->side)) != cudaSuccess) return status_of(e);
  }
  for (int b = 0; b < std::min(c, 2); ++b)
    if ((e = cudaStreamWaitEvent(st, ov->topk_done[b], 0)) != cudaSuccess) return status_of(e);
  lock.unlock();
  return mla_own_selection(q, kv, idx, T, S, H, k, q_pos0, sm_scale, out, lse, st);
}

size_t dsa_forward_fused_workspace_size(int T, int S, int Hi, int H, int k, int chunk) {
  (void)Hi;
  (void)H;
  if (T <= 0 || S <= 0 || k <= 0 || k > 2048 || S > kFusedMaxS) return 0;
  return fused_layout(T, S, k, chunk).total;
}

int dsa_forward_fused(const void* q8, const float* q_scale, const void* k8, const float* k_scale,
                      const float* w, const void* q, const void* kv, int T, int S, int Hi, int H,
                      int q_pos0, int k, int chunk, float scale, float sm_scale, int32_t* idx_out,
                      void* out, float* lse, void* workspace, size_t ws_bytes,
                      dsa_stream_t stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!q8 || !k8 || !w || !q || !kv || !out || T < 0 || S < 0 || q_pos0 < 0 || k <= 0 ||
      (k & 3) || !(scale > 0.f) || !(sm_scale > 0.f) || !aligned16(q8) || !aligned16(k8))
    return DSA_ERR_INVALID_ARG;
  if (!valid_hi(Hi)) return DSA_ERR_UNSUPPORTED;
  if (H < 1 || H > 128) return DSA_ERR_UNSUPPORTED;
  if (k > 2048 || S > kFusedMaxS) return DSA_ERR_UNSUPPORTED;
  if (T == 0) return DSA_OK;
  if (S == 0) return DSA_ERR_INVALID_ARG;
  const size_t need = dsa_forward_fused_workspace_size(T, S, Hi, H, k, chunk);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return DSA_ERR_WORKSPACE;
  const FusedLayout L = fused_layout(T, S, k, chunk);
  char* ws = static_cast<char*>(workspace);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + L.idx);
  if (!aligned16(idx)) return DSA_ERR_INVALID_ARG;
  unsigned* err = device_error_word();
  if (!err) return DSA_ERR_CUDA;
  const int rows = chunk <= 0 ? T : std::min(chunk, T);
  // the sampled keys (the first 256 of every 4096) in a compact cache: one
  // strided copy for the whole segments, one for the last, partial one
  uint8_t* k8s = reinterpret_cast<uint8_t*>(ws + L.k8s);
  float* kss = k_scale ? reinterpret_cast<float*>(ws + L.kss) : nullptr;
  const size_t full = static_cast<size_t>(S) / 4096;
  const size_t tail = std::min<size_t>(static_cast<size_t>(S) % 4096, 256);
  const uint8_t* k8b = static_cast<const uint8_t*>(k8);
  cudaError_t e = cudaSuccess;
  if (full > 0)
    e = cudaMemcpy2DAsync(k8s, 256 * 128, k8b, 4096 * 128, 256 * 128, full,
                          cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && tail > 0)
    e = cudaMemcpyAsync(k8s + full * 256 * 128, k8b + full * 4096 * 128, tail * 128,
                        cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && kss && full > 0)
    e = cudaMemcpy2DAsync(kss, 256 * 4, k_scale, 4096 * 4, 256 * 4, full,
                          cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && kss && tail > 0)
    e = cudaMemcpyAsync(kss + full * 256, k_scale + full * 4096, tail * 4,
                        cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws + L.fail_total, 0, 4, st);
  if (e != cudaSuccess) return status_of(e);
  // Per chunk c (buffers of parity b = c & 1): on the caller's stream the
  // sample pass, the thresholds and the filter pass; on the side stream the
  // select and recompute kernels, beside the next chunk's passes. The filter
  // pass of chunk c+2 rewrites buffers b, so it first waits for chunk c's
  // selection; the attention waits for every selection.
  std::unique_lock<std::mutex> lock(g_overlap_mu);
  Overlap* ov = L.nbuf == 2 ? overlap_for_current_device() : nullptr;
  if (!ov) lock.unlock();
  cudaStream_t side = ov ? ov->side : st;
  if (ov && ((e = cudaEventRecord(ov->start, st)) != cudaSuccess ||
             (e = cudaStreamWaitEvent(ov->side, ov->start, 0)) != cudaSuccess))
    return status_of(e);
  int c = 0;
  for (int c0 = 0; c0 < T; c0 += rows, ++c) {
    const int b = c & 1;
    const int n = std::min(rows, T - c0);
    const uint8_t* q8c = static_cast<const uint8_t*>(q8) + static_cast<size_t>(c0) * Hi * 128;
    const float* qsc = q_scale ? q_scale + c0 : nullptr;
    const float* wc = w + static_cast<size_t>(c0) * Hi;
    // 1. each row's scores against the sampled keys the chunk's last row sees
    const long long m_c =
        sample_count(static_cast<int>(std::min<long long>(static_cast<long long>(q_pos0) + c0 + n,
                                                          S)));
    IndexerArgs a;
    a.T = n;
    a.S = static_cast<int>(m_c);
    a.Hi = Hi;
    a.q_pos0 = q_pos0 + c0;
    a.scale = scale;
    a.w = wc;
    a.q_scale = qsc;
    a.k_scale = kss;
    a.scores = reinterpret_cast<float*>(ws + L.sample);
    a.ld = L.ldm;
    a.err = err;
    e = launch_indexer(a, q8c, k8s, m_c, st);
    // 2. the rows' thresholds
    FusedSelArgs F;
    F.T = n;
    F.S = S;
    F.q_pos0 = q_pos0 + c0;
    F.k = k;
    F.Hi = Hi;
    F.scale = scale;
    F.sample = a.scores;
    F.ld_sample = L.ldm;
    F.tau = reinterpret_cast<unsigned*>(ws + L.tau);
    F.cand_count = reinterpret_cast<unsigned*>(ws + L.cnt[b]);
    F.cand_key = reinterpret_cast<unsigned*>(ws + L.ckey[b]);
    F.cand_idx = reinterpret_cast<int*>(ws + L.cidx[b]);
    F.cand_cap = kFusedCandCap;
    F.fail_count = reinterpret_cast<unsigned*>(ws + L.fail[b]);
    F.fail_rows = reinterpret_cast<int*>(ws + L.fail[b]) + 1;
    F.fail_total = reinterpret_cast<unsigned*>(ws + L.fail_total);
    F.q8 = q8c;
    F.q_scale = qsc;
    F.k8 = k8b;
    F.k_scale = k_scale;
    F.w = wc;
    F.scratch = reinterpret_cast<float*>(ws + L.scratch);
    F.ld = L.ld;
    F.slots = kFusedSlots;
    F.idx = idx + static_cast<size_t>(c0) * k;
    F.err = err;
    if (e == cudaSuccess) e = launch_fused_tau(F, st);
    // 3. the filter-mode indexer: candidate lists instead of scores, into
    // buffers b once chunk c-2's selection has read them
    if (e == cudaSuccess && ov && c >= 2) e = cudaStreamWaitEvent(st, ov->topk_done[b], 0);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws + L.cnt[b], 0, static_cast<size_t>(n) * 4, st);
    IndexerArgs fa = a;
    fa.S = S;
    fa.k_scale = k_scale;
    fa.scores = nullptr;
    fa.ld = 0;
    fa.tau = F.tau;
    fa.cand_count = reinterpret_cast<unsigned*>(ws + L.cnt[b]);
    fa.cand_key = reinterpret_cast<unsigned*>(ws + L.ckey[b]);
    fa.cand_idx = reinterpret_cast<int*>(ws + L.cidx[b]);
    fa.cand_cap = kFusedCandCap;
    if (e == cudaSuccess) e = launch_indexer(fa, q8c, k8b, S, st);
    // 4. the exact selection among the candidates; 5. the rest recomputed
    if (e == cudaSuccess && ov) {
      e = cudaEventRecord(ov->idx_done[b], st);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(side, ov->idx_done[b], 0);
    }
    if (e == cudaSuccess) e = cudaMemsetAsync(ws + L.fail[b], 0, 4, side);
    if (e == cudaSuccess) e = launch_fused_select(F, side);
    if (e == cudaSuccess) e = launch_fused_fallback(F, side);
    if (e == cudaSuccess && ov) e = cudaEventRecord(ov->topk_done[b], side);
    if (e != cudaSuccess) return status_of(e);
  }
  if (ov) {
    for (int b = 0; b < std::min(c, 2); ++b)
      if ((e = cudaStreamWaitEvent(st, ov->topk_done[b], 0)) != cudaSuccess) return status_of(e);
    lock.unlock();
  }
  return mla_own_selection(q, kv, idx, T, S, H, k, q_pos0, sm_scale, out, lse,
                           static_cast<cudaStream_t>(stream));
}

int dsa_forward_fused_fallback_rows(const void* workspace, int T, int S, int k, int chunk,
                                    dsa_stream_t stream) {
  if (!workspace || T <= 0 || S <= 0 || k <= 0 || k > 2048 || S > kFusedMaxS)
    return DSA_ERR_INVALID_ARG;
  const FusedLayout L = fused_layout(T, S, k, chunk);
  unsigned v = 0;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess)
    e = cudaMemcpy(&v, static_cast<const char*>(workspace) + L.fail_total, sizeof v,
                   cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return status_of(e);
  return static_cast<int>(v);
}

size_t dsa_decode_paged_workspace_size(int B, int nq, int max_blocks, int Hi, int H, int k) {
  (void)Hi;
  (void)H;
  if (B <= 0 || nq <= 0 || max_blocks <= 0 || k <= 0) return 0;
  const size_t rows = static_cast<size_t>(B) * nq;
  return round_up(rows * max_blocks * 64 * sizeof(float), 256) +
         round_up(rows * k * sizeof(int32_t), 256);
}

int dsa_decode_paged(const void* q8, const float* q_scale, const float* w, const void* q,
                     const void* k8_pool, const float* k_scale_pool, const void* kv_pool,
                     const int32_t* block_table, const int32_t* seq_len, int B, int nq,
                     int max_blocks, int nblk, int Hi, int H, int k, float scale, float sm_scale,
                     int32_t* idx_out, void* out, float* lse, void* workspace, size_t ws_bytes,
                     dsa_stream_t stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!q8 || !w || !q || !k8_pool || !kv_pool || !block_table || !seq_len || !out || B < 0 ||
      nq < 1 || max_blocks < 1 || nblk < 1 || k <= 0 || (k & 3) || !(scale > 0.f) ||
      !(sm_scale > 0.f) || !aligned16(q8) || !aligned16(k8_pool) || !aligned16(kv_pool))
    return DSA_ERR_INVALID_ARG;
  if (!valid_hi(Hi) || nq * Hi > 256) return DSA_ERR_UNSUPPORTED;
  if (H < 1 || H > 128) return DSA_ERR_UNSUPPORTED;
  if (B == 0) return DSA_OK;
  const size_t need = dsa_decode_paged_workspace_size(B, nq, max_blocks, Hi, H, k);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return DSA_ERR_WORKSPACE;
  const int rows = B * nq;
  const int64_t ld = static_cast<int64_t>(max_blocks) * 64;
  float* scores = static_cast<float*>(workspace);
  int32_t* idx = idx_out;
  if (!idx)
    idx = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) +
                                     round_up(static_cast<size_t>(rows) * ld * 4, 256));
  if (!aligned16(idx)) return DSA_ERR_INVALID_ARG;

  IndexerArgs a;
  a.Hi = Hi;
  a.scale = scale;
  a.w = w;
  a.q_scale = q_scale;
  a.k_scale = k_scale_pool;
  a.scores = scores;
  a.ld = ld;
  a.block_table = block_table;
  a.max_blocks = max_blocks;
  a.nblk = nblk;
  a.seq_len = seq_len;
  a.nq = nq;
  a.B = B;
  a.max_ctx = max_blocks * 64;
  a.err = device_error_word();
  if (!a.err) return DSA_ERR_CUDA;
  int s = status_of(launch_indexer(a, q8, k8_pool, static_cast<long long>(nblk) * 64, st));
  if (s != DSA_OK) return s;
  s = run_topk(scores, rows, 0, ld, 0, seq_len, nq, k, idx, st);
  if (s != DSA_OK) return s;
  return mla_own_selection_paged(q, kv_pool, block_table, seq_len, idx, B, nq, max_blocks, nblk,
                                 H, k, sm_scale, out, lse, st);
}

}  // extern "C"

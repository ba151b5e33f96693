// dsa_internal.h -- launch interfaces between the C ABI (api.cu) and the
// kernels. Not installed; the public interface is include/dsa.h.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

namespace dsa {

struct IndexerArgs {
  int T = 0, S = 0, Hi = 0, q_pos0 = 0;   // prefill: query rows, keys, heads, first position
  float scale = 1.f;
  const float* w = nullptr;               // [queries][Hi]
  const float* q_scale = nullptr;         // [queries] or null
  const float* k_scale = nullptr;         // [keys] (contiguous) or [nblk*64] (paged) or null
  float* scores = nullptr;                // [queries][ld]
  long long ld = 0;
  // paged (decode) cache; block_table == nullptr selects the contiguous cache
  const int* block_table = nullptr;
  int max_blocks = 0, nblk = 0, nq = 1, B = 0, max_ctx = 0;
  const int* seq_len = nullptr;
  unsigned* err = nullptr;
  // filter mode (prefill): with tau set, no scores are written; every score
  // whose order key is >= tau[t] goes to row t's candidate list instead
  const unsigned* tau = nullptr;          // [T] order-key thresholds
  unsigned* cand_count = nullptr;         // [T], zero before the launch
  unsigned* cand_key = nullptr;           // [T][cand_cap]
  int* cand_idx = nullptr;                // [T][cand_cap]
  int cand_cap = 0;
  // filled in by launch_indexer
  int n_mma = 0, q_box_rows = 0, tmem_cols = 0, tiles_per_cta = 0;
};

struct TopkArgs {
  const float* scores = nullptr;
  long long ld = 0;
  int rows = 0, k = 0;
  int q_pos0 = 0, S = 0;                  // prefill row length min(q_pos0 + r + 1, S)
  const int* seq_len = nullptr;           // decode row length seq_len[r/nq] - nq + r%nq + 1
  int nq = 1;
  int* idx = nullptr;
  unsigned* err = nullptr;
  bool narrow = false;                    // 256-thread CTAs (beside the indexer)
};

// The prefill's selection without a score matrix in HBM: a threshold per row
// from the scores over the sampled keys, the filter-mode indexer's candidate
// lists, an exact select among them, and a CUDA-core recompute for the rows
// whose candidates miss [k, cand_cap].
struct FusedSelArgs {
  int T = 0, S = 0, q_pos0 = 0, k = 0, Hi = 0;
  float scale = 1.f;
  const float* sample = nullptr;          // [T][ld_sample] scores over the sampled keys
  long long ld_sample = 0;
  unsigned* tau = nullptr;                // [T] order-key thresholds
  const unsigned* cand_count = nullptr;   // [T]
  const unsigned* cand_key = nullptr;     // [T][cand_cap]
  const int* cand_idx = nullptr;          // [T][cand_cap]
  int cand_cap = 0;
  unsigned* fail_count = nullptr;         // [1], zero before the select
  unsigned* fail_total = nullptr;         // [1], rows sent to the recompute in the whole call
  int* fail_rows = nullptr;               // [T]
  // inputs of the recompute (rows of this call; keys of the whole cache)
  const uint8_t* q8 = nullptr;
  const float* q_scale = nullptr;
  const uint8_t* k8 = nullptr;
  const float* k_scale = nullptr;
  const float* w = nullptr;
  float* scratch = nullptr;               // [slots][ld] one score row per fallback CTA
  long long ld = 0;
  int slots = 0;
  int* idx = nullptr;                     // [T][k] out
  unsigned* err = nullptr;
};

struct ProjArgs {
  int T = 0, d = 0, Hi = 0, N = 0;        // tokens, hidden width, indexer heads, outputs
  const float* rope = nullptr;            // [T][64] (cos, sin) pairs
  float* y = nullptr;                     // workspace [T][Hi*128 + 128] fp32, rotated q | k
  long long ldy = 0;                      // row stride of y in the plain GEMM
  long long zstride = 0;                  // plain GEMM: offset of split z's output
  int kb = 0;                             // plain GEMM: B's K extent (0: d); B's K wraps
  int kt_split = 0;                       // plain GEMM: 64-wide K steps per split (0: all)
  unsigned* amax_q = nullptr;             // workspace [T], |y| maximum as float bits
  unsigned* amax_k = nullptr;
  float* a = nullptr;                     // [T][Hi] per-head weights out
  uint8_t* q8 = nullptr;                  // [T][Hi][128] e4m3 out
  uint8_t* k8 = nullptr;                  // [T][128] e4m3 out
  float* q_scale = nullptr;               // [T] out
  float* k_scale = nullptr;               // [T] out
  unsigned* err = nullptr;
};

struct IndexerBwdArgs {
  int T = 0, S = 0, Hi = 0, q_pos0 = 0;
  float scale = 1.f;
  const uint8_t* q8 = nullptr;            // [T][Hi][128] e4m3
  const float* q_scale = nullptr;         // [T] or null
  const uint8_t* k8 = nullptr;            // [S][128] e4m3
  const float* k_scale = nullptr;         // [S] or null
  const float* w = nullptr;               // [T][Hi]
  const float* grad = nullptr;            // [T][ldg] dL/dI
  long long ldg = 0;
  float* dq = nullptr;                    // [T][Hi][128] out
  float* dk = nullptr;                    // [S][128] out
  float* dw = nullptr;                    // [T][Hi] out
};

struct MlaArgs {
  int T = 0, S = 0, H = 0, k = 0;         // query rows, keys (contiguous), heads, slots per row
  float sm_scale_log2 = 0.f;              // sm_scale * log2(e)
  const int* idx = nullptr;               // [T][k] (unused in dense mode)
  // dense causal mode: row r's slots are every key it sees, 0 .. its position
  // (q_pos0 + r, or the paged query's position); no index sets are read
  int dense = 0, q_pos0 = 0;
  // the index sets hold their selected slots first (the library's own
  // top-k): a row walks only min(k, keys it sees) slots, since the rest are
  // -1. Row r of a contiguous cache sits at position q_pos0 + r.
  int compact = 0;
  const int* block_table = nullptr;       // paged cache (decode) or null
  int max_blocks = 0, nblk = 0, nq = 1;
  const int* seq_len = nullptr;
  __nv_bfloat16* out = nullptr;           // [T][H][512]
  float* lse = nullptr;                   // [T][H] or null
  const __nv_bfloat16* kv = nullptr;      // [kv_rows][576] (filled by the launcher)
  int kv_rows = 0;                        // rows of the kv tensor map (filled by the launcher)
  unsigned* err = nullptr;
};

// 2D tensor map: `rows` rows of `inner` elements, `row_stride` bytes apart.
cudaError_t make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         uint64_t inner, uint64_t rows, uint64_t row_stride, uint32_t box_inner,
                         uint32_t box_rows, CUtensorMapSwizzle swizzle);

cudaError_t launch_indexer(const IndexerArgs& a, const void* q8, const void* k8, long long k_rows,
                           cudaStream_t st);
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st);
cudaError_t launch_fused_tau(const FusedSelArgs& a, cudaStream_t st);
cudaError_t launch_fused_select(const FusedSelArgs& a, cudaStream_t st);
cudaError_t launch_fused_fallback(const FusedSelArgs& a, cudaStream_t st);
constexpr int kFusedCandCap = 4096;       // candidates per row
constexpr int kFusedSlots = 148;          // fallback CTAs (one score row each)
constexpr int kFusedMaxS = 131072;        // longest row the fused selection takes
cudaError_t launch_window(int T, int S, int q_pos0, int window, int k, int* idx, cudaStream_t st);
cudaError_t launch_project(const ProjArgs& a, const void* h, const void* wt, cudaStream_t st);
// C [M][ldc] fp32 = A [M][K] x B [N][K]^T, bf16 operands, K a multiple of 8.
cudaError_t launch_gemm_f32(const void* a, const void* b, float* c, int M, int N, int K,
                            long long ldc, unsigned* err, cudaStream_t st, int kb = 0,
                            int kt_split = 0);
cudaError_t launch_attention_probs(const void* q, const void* kv, const float* lse, int T, int S,
                                   int H, int q_pos0, float sm_scale, float* p, long long ldp,
                                   float* z, long long ldz, unsigned* err, cudaStream_t st);
cudaError_t launch_indexer_kl(const float* I, long long ldi, const float* p, long long ldp, int T,
                              int S, int q_pos0, float* loss, float* grad, long long ldg,
                              cudaStream_t st);
size_t indexer_backward_workspace(int T, int S, int Hi);
cudaError_t launch_indexer_backward(const IndexerBwdArgs& a, void* workspace, unsigned* err,
                                    cudaStream_t st);
cudaError_t launch_sparse_mla(const MlaArgs& a, const void* q, const void* kv, long long kv_rows,
                              long long q_rows, cudaStream_t st);

int indexer_queries_per_cta(int Hi);

// Records a message for dsa_last_error_string() on this thread.
void set_last_error(const char* msg);

}  // namespace dsa

// topk.cu -- per-query top-k selection over score rows.
//
// Step 3 of the four-step workflow ("DeepSeek-V3.2-Exp 模型优势与 DSA 工作原理",
// section 4): each query keeps its k highest-scoring keys, or every key when
// it sees at most k of them (page 3, section 2 "风险边界明确"). Ties are
// broken by the smaller key index, which makes the selected set unique.
//
// One CTA per row. Scores map to order-preserving 32-bit keys; a radix
// select with three histogram passes (11 + 11 + 10 bits, shared-memory
// histograms) finds the k-th largest key T and how many keys equal to T
// are still needed. A last pass walks the row in index order with a
// block-wide scan and writes every index whose key is > T plus the first
// `need` indices whose key == T. The output is therefore sorted by index.
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kTopkThreads = 512;
constexpr int kWarps = kTopkThreads / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ long long row_length(const TopkArgs& a, int r) {
  if (a.seq_len) {
    const int b = r / a.nq, j = r % a.nq;
    return static_cast<long long>(a.seq_len[b]) - a.nq + j + 1;
  }
  return min(static_cast<long long>(a.q_pos0) + r + 1, static_cast<long long>(a.S));
}

// Inclusive prefix sum over a warp.
__device__ __forceinline__ unsigned warp_incl_scan(unsigned v) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned n = __shfl_up_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) >= o) v += n;
  }
  return v;
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const TopkArgs a) {
  __shared__ unsigned hist[2048];
  __shared__ unsigned warp_tot[kWarps];
  __shared__ unsigned s_bucket, s_above;
  const int r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int* out = a.idx + static_cast<long long>(r) * a.k;
  long long n = row_length(a, r);
  if (n < 0) n = 0;
  if (n > a.ld) {                       // cannot happen for validated calls
    if (tid == 0) raise_error(a.err, kErrBounds);
    n = a.ld;
  }
  if (n <= a.k) {                       // short context: every key
    for (int j = tid; j < a.k; j += kTopkThreads) out[j] = j < n ? j : -1;
    return;
  }
  const float* x = a.scores + static_cast<long long>(r) * a.ld;
  const float4* x4 = reinterpret_cast<const float4*>(x);
  const long long n4 = (n + 3) >> 2;

  // ----------------------------------------------------- radix select
  uint32_t prefix = 0;                  // key bits fixed so far
  unsigned want = static_cast<unsigned>(a.k);   // rank still to find within the prefix
  const int bits[3] = {11, 11, 10};
  int shift = 32;
  for (int p = 0; p < 3; ++p) {
    const int nb = 1 << bits[p];
    shift -= bits[p];
    for (int i = tid; i < nb; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    const int hi_shift = shift + bits[p];
    for (long long i = tid; i < n4; i += kTopkThreads) {
      const float4 v = x4[i];
      const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (4 * i + c >= n) break;
        const uint32_t u = order_key(e[c]);
        if (p == 0 || (u >> hi_shift) == prefix)
          atomicAdd(&hist[(u >> shift) & (nb - 1)], 1u);
      }
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins [top - per*l - per + 1, top - per*l], scanned from the top
      const int per = nb / 32;
      const int top = nb - 1 - lane * per;
      unsigned local = 0;
      for (int j = 0; j < per; ++j) local += hist[top - j];
      const unsigned incl = warp_incl_scan(local);
      const unsigned excl = incl - local;
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= want);
      const int first = __ffs(hit) - 1;
      if (lane == first) {
        unsigned cum = excl;
        for (int j = 0; j < per; ++j) {
          const unsigned c = hist[top - j];
          if (cum + c >= want) {
            s_bucket = top - j;
            s_above = cum;
            break;
          }
          cum += c;
        }
      }
    }
    __syncthreads();
    prefix = (prefix << bits[p]) | s_bucket;
    want -= s_above;
    __syncthreads();
  }
  const uint32_t thr = prefix;          // k-th largest key
  const unsigned need = want;           // keys == thr to take, smallest indices first

  // ------------------------------------------- ordered final selection
  unsigned base_sel = 0, base_eq = 0;
  for (long long i0 = 0; i0 < n4; i0 += kTopkThreads) {
    const long long i = i0 + tid;
    unsigned gt_mask = 0, eq_mask = 0;
    if (i < n4) {
      const float4 v = x4[i];
      const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (4 * i + c < n) {
          const uint32_t u = order_key(e[c]);
          gt_mask |= (u > thr) << c;
          eq_mask |= (u == thr) << c;
        }
      }
    }
    // exclusive scan of (eq count) to rank equal keys in index order
    const unsigned n_eq = __popc(eq_mask);
    unsigned incl = warp_incl_scan(n_eq);
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    unsigned wbase = 0, total = 0;
    for (int w = 0; w < kWarps; ++w) {
      const unsigned t = warp_tot[w];
      if (w < warp) wbase += t;
      total += t;
    }
    unsigned eq_rank = base_eq + wbase + incl - n_eq;
    unsigned sel_mask = gt_mask;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (eq_mask & (1u << c)) {
        if (eq_rank < need) sel_mask |= 1u << c;
        ++eq_rank;
      }
    }
    base_eq += total;
    __syncthreads();
    const unsigned n_sel = __popc(sel_mask);
    incl = warp_incl_scan(n_sel);
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    wbase = 0;
    total = 0;
    for (int w = 0; w < kWarps; ++w) {
      const unsigned t = warp_tot[w];
      if (w < warp) wbase += t;
      total += t;
    }
    unsigned pos = base_sel + wbase + incl - n_sel;
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (sel_mask & (1u << c)) {
        if (pos < static_cast<unsigned>(a.k)) out[pos] = static_cast<int>(4 * i + c);
        ++pos;
      }
    base_sel += total;
    __syncthreads();
  }
  if (tid == 0 && base_sel != static_cast<unsigned>(a.k)) raise_error(a.err, kErrBounds);
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st) {
  if (a.rows <= 0) return cudaSuccess;
  topk_kernel<<<a.rows, kTopkThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa

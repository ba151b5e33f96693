// topk_impl.cuh -- per-query top-k selection over score rows.
//
// Compiled as 512-thread CTAs (topk.cu: rows that have the GPU to
// themselves) and as 256-thread CTAs (topk_narrow.cu: the chunks of a prefill,
// whose selection runs on a side stream while the next chunk's indexer runs,
// taking SMs as the indexer's CTAs retire); fused_topk.cu uses its device
// functions only. The including
// file defines DSA_TOPK_THREADS and DSA_TOPK_MIN_CTAS, and DSA_TOPK_LAUNCH,
// the name of the row-per-CTA kernel's launcher, where it wants that kernel.
//
// Step 3 of the four-step workflow ("DeepSeek-V3.2-Exp 模型优势与 DSA 工作原理",
// section 4): each query keeps its k highest-scoring keys, or every key when
// it sees at most k of them (page 3, section 2 "风险边界明确"). Ties are
// broken by the smaller key index, which makes the selected set unique.
//
// One CTA per row. Scores map to order-preserving 32-bit keys.
//   pass 1: a 4096-bin histogram of the top 12 key bits locates the bucket
//           holding the k-th largest key;
//   pass 2: one ordered sweep of the row (block-wide scans) appends every
//           index above that bucket to a "sure" list and every member of the
//           bucket (key, index) to a candidate list, both in index order;
//   then, in shared memory only, a two-level radix select on the low 20 bits
//   picks the candidates still needed (ties to the first in index order) and
//   the two index-sorted lists are merged into the output.
// Rows whose bucket holds more candidates than the buffer, or calls with
// k > 4096, take the general path: three histogram passes over the row and
// an ordered selection pass. Either way the output is sorted by index.
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kTopkThreads = DSA_TOPK_THREADS;
constexpr int kWarps = kTopkThreads / 32;
constexpr int kBins = 4096;          // 12-bit first-level histogram
constexpr int kFastMaxK = 4096;      // capacity of the "sure" list
constexpr int kCandCap = 4096;       // capacity of the bucket's candidate list

struct TopkSmem {
  unsigned hist[kBins];              // also the chosen-candidate list after pass 2
  int sure[kFastMaxK];
  unsigned cand_key[kCandCap];       // low 20 key bits
  int cand_idx[kCandCap];
  unsigned warp_tot[kWarps];
  unsigned s_bucket, s_above;
  unsigned s_count;
};

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

__device__ __forceinline__ unsigned warp_incl_scan(unsigned v) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned n = __shfl_up_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) >= o) v += n;
  }
  return v;
}

// Exclusive prefix sum over the block; `total` gets the block sum. Two syncs.
__device__ __forceinline__ unsigned block_excl_scan(unsigned v, unsigned* warp_tot,
                                                    unsigned& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned incl = warp_incl_scan(v);
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  unsigned base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const unsigned t = warp_tot[w];
    base += (w < warp) ? t : 0u;
    tot += t;
  }
  __syncthreads();
  total = tot;
  return base + incl - v;
}

// With hist[0..nb) filled, find (from the top) the bucket where the count
// reaches `want`; writes the bucket and the count strictly above it. Thread t
// sums bins [nb - (t+1)·per, nb - t·per); a block scan over those sums, taken
// from the top, tells which thread's range holds the bucket.
__device__ __forceinline__ void find_bucket(const unsigned* hist, int nb, unsigned want,
                                            unsigned* s_bucket, unsigned* s_above) {
  __shared__ unsigned scan_tot[kWarps];
  const int tid = threadIdx.x;
  const int per = nb / kTopkThreads > 0 ? nb / kTopkThreads : 1;
  const int top = nb - 1 - tid * per;            // this thread's highest bin
  unsigned local = 0;
  if (top >= 0)
    for (int j = 0; j < per; ++j) local += hist[top - j];
  unsigned tot;
  const unsigned excl = block_excl_scan(local, scan_tot, tot);
  if (top >= 0 && excl < want && excl + local >= want) {
    unsigned cum = excl;
    for (int j = 0; j < per; ++j) {
      const unsigned c = hist[top - j];
      if (cum + c >= want) {
        *s_bucket = top - j;
        *s_above = cum;
        break;
      }
      cum += c;
    }
  }
  __syncthreads();
}

// Writes the row's selection in index order: every key whose order key is
// above `thr`, plus the first `need` keys equal to `thr`.
__device__ void write_selection(const float4* x4, long long n, long long n4, uint32_t thr,
                                unsigned need, int* out, int k, TopkSmem& sm) {
  const int tid = threadIdx.x;
  unsigned base_gt = 0, base_eq = 0;
  for (long long i0 = 0; i0 < n4; i0 += kTopkThreads) {
    const long long i = i0 + tid;
    unsigned gt_m = 0, eq_m = 0;
    if (i < n4) {
      const float4 v = x4[i];
      const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (4 * i + c < n) {
          const uint32_t u = order_key(e[c]);
          gt_m |= static_cast<unsigned>(u > thr) << c;
          eq_m |= static_cast<unsigned>(u == thr) << c;
        }
    }
    unsigned tot;
    const unsigned ex = block_excl_scan(__popc(gt_m) | (__popc(eq_m) << 16), sm.warp_tot, tot);
    unsigned gt_before = base_gt + (ex & 0xffffu), eq_before = base_eq + (ex >> 16);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (gt_m & (1u << c)) {
        const unsigned p = gt_before + min(eq_before, need);
        if (p < static_cast<unsigned>(k)) out[p] = static_cast<int>(4 * i + c);
        ++gt_before;
      } else if (eq_m & (1u << c)) {
        if (eq_before < need) {
          const unsigned p = gt_before + eq_before;
          if (p < static_cast<unsigned>(k)) out[p] = static_cast<int>(4 * i + c);
        }
        ++eq_before;
      }
    }
    base_gt += tot & 0xffffu;
    base_eq += tot >> 16;
  }
}

// General path: 11 + 11 + 10-bit radix select over the row, then the ordered
// selection pass.
__device__ void select_general(const float4* x4, long long n, long long n4, int k, int* out,
                               TopkSmem& sm) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0;
  unsigned want = static_cast<unsigned>(k);
  const int bits[3] = {11, 11, 10};
  int shift = 32;
#pragma unroll
  for (int p = 0; p < 3; ++p) {
    const int nb = 1 << bits[p];
    shift -= bits[p];
    const int hi_shift = shift + bits[p];
    for (int i = tid; i < nb; i += kTopkThreads) sm.hist[i] = 0;
    __syncthreads();
    for (long long i = tid; i < n4; i += kTopkThreads) {
      const float4 v = x4[i];
      const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (4 * i + c >= n) break;
        const uint32_t u = order_key(e[c]);
        if (p == 0 || (u >> hi_shift) == prefix) atomicAdd(&sm.hist[(u >> shift) & (nb - 1)], 1u);
      }
    }
    __syncthreads();
    find_bucket(sm.hist, nb, want, &sm.s_bucket, &sm.s_above);
    prefix = (prefix << bits[p]) | sm.s_bucket;
    want -= sm.s_above;
    __syncthreads();
  }
  write_selection(x4, n, n4, prefix, want, out, k, sm);
}

// Number of entries of the ascending array a[0..m) that are below v.
__device__ __forceinline__ int count_below(const int* a, int m, int v) {
  int lo = 0, hi = m;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Fast path: the bucket `b` of the top 12 bits holds the k-th key; `above`
// keys lie in higher buckets.
__device__ void select_fast(const float4* x4, long long n, long long n4, int k, int* out,
                            TopkSmem& sm, unsigned b, unsigned above) {
  const int tid = threadIdx.x;
  const unsigned want = static_cast<unsigned>(k) - above;   // still needed from the bucket
  // pass 2: ordered sweep collecting the sure keys and the bucket's members
  unsigned base_sure = 0, base_cand = 0;
  for (long long i0 = 0; i0 < n4; i0 += kTopkThreads) {
    const long long i = i0 + tid;
    unsigned sure_m = 0, cand_m = 0;
    uint32_t keys[4] = {0, 0, 0, 0};
    if (i < n4) {
      const float4 v = x4[i];
      const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (4 * i + c < n) {
          const uint32_t u = order_key(e[c]);
          keys[c] = u;
          sure_m |= static_cast<unsigned>((u >> 20) > b) << c;
          cand_m |= static_cast<unsigned>((u >> 20) == b) << c;
        }
    }
    unsigned tot;
    const unsigned ex = block_excl_scan(__popc(sure_m) | (__popc(cand_m) << 16), sm.warp_tot, tot);
    unsigned ps = base_sure + (ex & 0xffffu), pc = base_cand + (ex >> 16);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (sure_m & (1u << c)) sm.sure[ps++] = static_cast<int>(4 * i + c);
      if (cand_m & (1u << c)) {
        sm.cand_key[pc] = keys[c] & 0xfffffu;
        sm.cand_idx[pc] = static_cast<int>(4 * i + c);
        ++pc;
      }
    }
    base_sure += tot & 0xffffu;
    base_cand += tot >> 16;
  }
  __syncthreads();
  const int ncand = static_cast<int>(base_cand);
  // radix select on the low 20 bits, inside shared memory (10 + 10 bits)
  for (int j = tid; j < 1024; j += kTopkThreads) sm.hist[j] = 0;
  __syncthreads();
  for (int j = tid; j < ncand; j += kTopkThreads) atomicAdd(&sm.hist[sm.cand_key[j] >> 10], 1u);
  __syncthreads();
  find_bucket(sm.hist, 1024, want, &sm.s_bucket, &sm.s_above);
  const unsigned bA = sm.s_bucket;
  const unsigned want2 = want - sm.s_above;
  __syncthreads();
  for (int j = tid; j < 1024; j += kTopkThreads) sm.hist[j] = 0;
  __syncthreads();
  for (int j = tid; j < ncand; j += kTopkThreads)
    if ((sm.cand_key[j] >> 10) == bA) atomicAdd(&sm.hist[sm.cand_key[j] & 1023u], 1u);
  __syncthreads();
  find_bucket(sm.hist, 1024, want2, &sm.s_bucket, &sm.s_above);
  const uint32_t thr = (bA << 10) | sm.s_bucket;
  const unsigned need = want2 - sm.s_above;
  __syncthreads();
  // chosen candidates, compacted in index order into list2 (reusing hist)
  int* list2 = reinterpret_cast<int*>(sm.hist);
  unsigned base_gt = 0, base_eq = 0;
  for (int j0 = 0; j0 < ncand; j0 += kTopkThreads) {
    const int j = j0 + tid;
    const bool in = j < ncand;
    const uint32_t key = in ? sm.cand_key[j] : 0u;
    const bool gt = in && key > thr, eq = in && key == thr;
    unsigned tot;
    const unsigned ex = block_excl_scan(static_cast<unsigned>(gt) | (static_cast<unsigned>(eq) << 16),
                                        sm.warp_tot, tot);
    const unsigned gt_before = base_gt + (ex & 0xffffu), eq_before = base_eq + (ex >> 16);
    if (gt) list2[gt_before + min(eq_before, need)] = sm.cand_idx[j];
    else if (eq && eq_before < need) list2[gt_before + eq_before] = sm.cand_idx[j];
    base_gt += tot & 0xffffu;
    base_eq += tot >> 16;
  }
  __syncthreads();
  // merge the two index-sorted lists (disjoint) into the output
  const int na = static_cast<int>(above), nb2 = static_cast<int>(want);
  for (int i = tid; i < na; i += kTopkThreads) {
    const int v = sm.sure[i];
    out[i + count_below(list2, nb2, v)] = v;
  }
  for (int j = tid; j < nb2; j += kTopkThreads) {
    const int v = list2[j];
    out[j + count_below(sm.sure, na, v)] = v;
  }
}

// Radix select in shared memory over keys[0..m). With kPasses = 3 (11 + 11 +
// 10 bits) it returns the `want`-th largest key and how many keys equal to it
// rank within the first `want`. With kPasses = 2 (12 + 10 bits) it returns
// the lower edge of the 22-bit bucket that holds the `want`-th largest key: a
// threshold at or below it, at least `want` keys at or above it. `hist` needs
// 2048 (3 passes) or 4096 (2 passes) entries and must not overlap `keys`.
template <int kPasses>
__device__ void smem_select(const uint32_t* keys, int m, unsigned want, unsigned* hist,
                            TopkSmem& sm, uint32_t* kth, unsigned* need) {
  const int tid = threadIdx.x;
  const int bits[3] = {kPasses == 3 ? 11 : 12, kPasses == 3 ? 11 : 10, 10};
  uint32_t prefix = 0;
  int shift = 32;
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int nb = 1 << bits[p];
    shift -= bits[p];
    const int hi_shift = shift + bits[p];
    for (int j = tid; j < nb; j += kTopkThreads) hist[j] = 0;
    __syncthreads();
    for (int j = tid; j < m; j += kTopkThreads) {
      const uint32_t u = keys[j];
      if (p == 0 || (u >> hi_shift) == prefix) atomicAdd(&hist[(u >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    find_bucket(hist, nb, want, &sm.s_bucket, &sm.s_above);
    prefix = (prefix << bits[p]) | sm.s_bucket;
    want -= sm.s_above;
    __syncthreads();
  }
  *kth = prefix << shift;
  *need = want;
}

// Ordered scan of a bitmap of n bits (bit i = key i): calls emit(rank, i) for
// every set bit, rank counting set bits in index order from 0.
template <typename F>
__device__ void bitmap_scan(const unsigned* bm, long long n, TopkSmem& sm, F emit) {
  const int tid = threadIdx.x;
  const int words = static_cast<int>((n + 31) >> 5);
  const int per = (words + kTopkThreads - 1) / kTopkThreads;
  const int w0 = min(words, tid * per), w1 = min(words, w0 + per);
  unsigned cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(bm[w]);
  unsigned tot;
  unsigned rank = block_excl_scan(cnt, sm.warp_tot, tot);
  for (int w = w0; w < w1; ++w) {
    unsigned b = bm[w];
    while (b) {
      const int bit = __ffs(b) - 1;
      emit(rank++, 32 * w + bit);
      b &= b - 1;
    }
  }
}

// With every key of a row of n (n <= kSampledMaxN) at or above some
// threshold in sm.cand_key / sm.cand_idx (ncand of them, any order, at least
// k): the k largest, ties to the smaller index, written to out in index
// order. An exact select in shared memory gives the k-th largest key and how
// many of its ties to take; two bitmaps of the row (above it / equal to it)
// and ordered scans put the selection in index order.
__device__ void select_from_candidates(long long n, int k, int ncand, int* out, TopkSmem& sm) {
  const int tid = threadIdx.x;
  uint32_t thr;
  unsigned need;
  smem_select<3>(sm.cand_key, ncand, static_cast<unsigned>(k), sm.hist, sm, &thr, &need);
  unsigned* gt = sm.hist;
  unsigned* eq = reinterpret_cast<unsigned*>(sm.sure);
  const int words = static_cast<int>((n + 31) >> 5);
  for (int w = tid; w < words; w += kTopkThreads) {
    gt[w] = 0u;
    eq[w] = 0u;
  }
  __syncthreads();
  for (int j = tid; j < ncand; j += kTopkThreads) {
    const uint32_t u = sm.cand_key[j];
    const int ix = sm.cand_idx[j];
    if (u > thr) atomicOr(&gt[ix >> 5], 1u << (ix & 31));
    else if (u == thr) atomicOr(&eq[ix >> 5], 1u << (ix & 31));
  }
  __syncthreads();
  // the first `need` ties in index order join the selection
  bitmap_scan(eq, n, sm, [&](unsigned r, int ix) {
    if (r < need) atomicOr(&gt[ix >> 5], 1u << (ix & 31));
  });
  __syncthreads();
  bitmap_scan(gt, n, sm, [&](unsigned r, int ix) {
    if (r < static_cast<unsigned>(k)) out[r] = ix;
  });
}

// Sampled path. The k-th largest key is estimated from a sample of the row
// (the first 256 keys of every 4096) with a margin; one sweep then keeps
// every key at or above the estimate, appended in any order with one shared
// atomic per warp. If at least k were kept, the selection lies among them,
// ties included (the k-th largest key is at or above the estimate): it is
// chosen exactly in shared memory and put back in index order through a
// bitmap of the row. Otherwise, or when the kept keys overflow the buffer,
// the caller falls back to the two-pass paths. Returns whether the selection
// was written.
constexpr int kSampleSeg = 4096;       // row segment
constexpr int kSampleRun = 256;        // sampled keys at the start of each segment
constexpr long long kSampledMaxN = 32ll * kSampleSeg;   // sample and bitmaps fit hist + sure

__device__ bool select_sampled(const float4* x4, long long n, long long n4, int k, int* out,
                               TopkSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int nseg = static_cast<int>((n + kSampleSeg - 1) / kSampleSeg);
  uint32_t* samp = sm.hist;                     // hist and sure are contiguous: 8192 keys
  // all of a thread's sample loads are issued before any is used
  const int runs4 = kSampleRun / 4;
  constexpr int kIters = (static_cast<int>(kSampledMaxN / kSampleSeg) * kSampleRun / 4) /
                         kTopkThreads;
  float4 sv[kIters];
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int j = tid + it * kTopkThreads;
    const long long i4 = static_cast<long long>(j / runs4) * (kSampleSeg / 4) + (j % runs4);
    sv[it] = (j < nseg * runs4 && i4 < n4) ? x4[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const int j = tid + it * kTopkThreads;
    if (j >= nseg * runs4) break;
    const long long i4 = static_cast<long long>(j / runs4) * (kSampleSeg / 4) + (j % runs4);
    const float e[4] = {sv[it].x, sv[it].y, sv[it].z, sv[it].w};
#pragma unroll
    for (int c = 0; c < 4; ++c)           // past the row end: 0, below every real key
      samp[4 * j + c] = (4 * i4 + c < n) ? order_key(e[c]) : 0u;
  }
  if (tid == 0) sm.s_count = 0;
  __syncthreads();
  const long long m = (n / kSampleSeg) * kSampleRun + min(static_cast<long long>(kSampleRun),
                                                           n % kSampleSeg);
  const long long rank = static_cast<long long>(1.4 * k * static_cast<double>(m) / n) + 9;
  if (rank >= m) return false;
  uint32_t tau;
  unsigned unused;
  smem_select<2>(samp, nseg * kSampleRun, static_cast<unsigned>(rank),
                 reinterpret_cast<unsigned*>(sm.cand_key), sm, &tau, &unused);
  // the sweep: keys >= tau appended with one atomic per warp and slot; four
  // 16-B loads per thread are issued before any is used
  constexpr int kBatch = 4;
  for (long long i0 = 0; i0 < n4; i0 += kTopkThreads * kBatch) {
    float4 v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const long long i = i0 + u * kTopkThreads + tid;
      v[u] = i < n4 ? x4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const long long i = i0 + u * kTopkThreads + tid;
      const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const bool in = i < n4 && 4 * i + c < n;
        const uint32_t key = order_key(e[c]);
        const bool keep = in && key >= tau;
        const unsigned ball = __ballot_sync(0xffffffffu, keep);
        if (ball) {
          unsigned base = 0;
          if (lane == 0) base = atomicAdd(&sm.s_count, static_cast<unsigned>(__popc(ball)));
          base = __shfl_sync(0xffffffffu, base, 0);
          if (keep) {
            const unsigned pos = base + __popc(ball & ((1u << lane) - 1u));
            if (pos < static_cast<unsigned>(kCandCap)) {
              sm.cand_key[pos] = key;
              sm.cand_idx[pos] = static_cast<int>(4 * i + c);
            }
          }
        }
      }
    }
  }
  __syncthreads();
  const unsigned kept = sm.s_count;
  if (kept < static_cast<unsigned>(k) || kept > static_cast<unsigned>(kCandCap)) return false;
  select_from_candidates(n, k, static_cast<int>(kept), out, sm);
  return true;
}

// The selection of one row of n scores (k of them, sorted by index, -1
// padded): every key when n <= k, else the sampled path, falling back to the
// two-pass paths.
__device__ void select_row(const float* row, long long n, int k, int* out, TopkSmem& sm) {
  const int tid = threadIdx.x;
  if (n <= k) {                         // short context: every key
    for (int j = tid; j < k; j += kTopkThreads) out[j] = j < n ? j : -1;
    return;
  }
  const float4* x4 = reinterpret_cast<const float4*>(row);
  const long long n4 = (n + 3) >> 2;
  if (k <= 2048 && n >= 4ll * k && n <= kSampledMaxN && select_sampled(x4, n, n4, k, out, sm))
    return;
  __syncthreads();
  // pass 1: 12-bit histogram of the whole row
  for (int i = tid; i < kBins; i += kTopkThreads) sm.hist[i] = 0;
  __syncthreads();
#pragma unroll 2
  for (long long i = tid; i < n4; i += kTopkThreads) {
    const float4 v = x4[i];
    const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (4 * i + c < n) atomicAdd(&sm.hist[order_key(e[c]) >> 20], 1u);
  }
  __syncthreads();
  find_bucket(sm.hist, kBins, static_cast<unsigned>(k), &sm.s_bucket, &sm.s_above);
  const unsigned b = sm.s_bucket, above = sm.s_above, in_bucket = sm.hist[b];
  __syncthreads();
  if (k <= kFastMaxK && in_bucket <= static_cast<unsigned>(kCandCap))
    select_fast(x4, n, n4, k, out, sm, b, above);
  else
    select_general(x4, n, n4, k, out, sm);
}

#ifdef DSA_TOPK_LAUNCH
__global__ void __launch_bounds__(kTopkThreads, DSA_TOPK_MIN_CTAS) topk_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  const int r = blockIdx.x;
  int* out = a.idx + static_cast<long long>(r) * a.k;
  long long n = row_length(a, r);
  if (n < 0) n = 0;
  if (n > a.ld) {                       // cannot happen for validated calls
    if (threadIdx.x == 0) raise_error(a.err, kErrBounds);
    n = a.ld;
  }
  select_row(a.scores + static_cast<long long>(r) * a.ld, n, a.k, out, sm);
}
#endif

}  // namespace

#ifdef DSA_TOPK_LAUNCH
cudaError_t DSA_TOPK_LAUNCH(const TopkArgs& a, cudaStream_t st) {
  if (a.rows <= 0) return cudaSuccess;
  const size_t smem = sizeof(TopkSmem);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  // the whole shared carveout, so shared memory never keeps a CTA off an SM
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  topk_kernel<<<a.rows, kTopkThreads, smem, st>>>(a);
  return cudaGetLastError();
}
#endif

}  // namespace dsa

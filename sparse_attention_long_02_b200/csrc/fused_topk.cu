// fused_topk.cu -- the prefill's top-k without a score matrix in HBM.
//
// Per chunk of query rows (the selection itself is that of topk_impl.cuh):
//   1. the indexer scores every row against the sampled keys only (the first
//      256 of every 4096, gathered into a compact cache);
//   2. tau_kernel: per row, the (1.4 k m / n + 9)-th largest of its m sampled
//      scores is a threshold with, in expectation, about 1.4 k of the row's n
//      keys at or above it;
//   3. the indexer in filter mode appends every (key, score) at or above the
//      threshold to the row's candidate list instead of writing scores;
//   4. select_kernel: with k to kFusedCandCap candidates, the k largest (ties
//      to the smaller index) are exactly among them, and are chosen in shared
//      memory; other rows go to a list;
//   5. fallback_kernel: each listed row's scores are recomputed on CUDA cores
//      into a scratch row and selected by the full top-k. The list is empty
//      for all but rare rows; the kernel then returns at once.
#define DSA_TOPK_THREADS 512
#define DSA_TOPK_MIN_CTAS 1
#include "topk_impl.cuh"

#include <cuda_fp8.h>

namespace dsa {
namespace {

// Compact index of key position p among the sampled keys.
__device__ __forceinline__ long long sample_index(long long p) {
  return (p >> 12) * kSampleRun + min(p & (kSampleSeg - 1), static_cast<long long>(kSampleRun - 1));
}

__device__ __forceinline__ long long row_pos(const FusedSelArgs& A, int r) {
  return min(static_cast<long long>(A.q_pos0) + r, static_cast<long long>(A.S) - 1);
}

__global__ void __launch_bounds__(kTopkThreads, 1) tau_kernel(const FusedSelArgs A) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  const int r = blockIdx.x, tid = threadIdx.x;
  const long long pos = row_pos(A, r), n = pos + 1;
  if (n <= A.k) {                       // every key: no candidates needed
    if (tid == 0) A.tau[r] = 0xffffffffu;
    return;
  }
  // the row's sampled scores, at most 8192 of them in shared memory (runs of
  // 256 taken every `stride` runs when the row is longer than 131072)
  const long long m_all = sample_index(pos) + 1;
  const long long runs = (m_all + kSampleRun - 1) / kSampleRun;
  const long long stride = (runs * kSampleRun + 8191) / 8192;
  const long long used = (runs + stride - 1) / stride;
  const long long last = (used - 1) * stride;
  const int m = static_cast<int>((used - 1) * kSampleRun +
                                 min(static_cast<long long>(kSampleRun), m_all - last * kSampleRun));
  uint32_t* samp = sm.hist;             // hist and sure are contiguous: 8192 keys
  const float* row = A.sample + static_cast<long long>(r) * A.ld_sample;
  for (int e = tid; e < m; e += kTopkThreads) {
    const long long j = (e / kSampleRun) * stride * kSampleRun + e % kSampleRun;
    samp[e] = order_key(row[j]);
  }
  __syncthreads();
  const long long rank = static_cast<long long>(1.4 * A.k * static_cast<double>(m) / n) + 9;
  uint32_t tau = 0;                     // too few samples: keep every key
  if (rank < m) {
    unsigned unused;
    smem_select<2>(samp, m, static_cast<unsigned>(rank), reinterpret_cast<unsigned*>(sm.cand_key),
                   sm, &tau, &unused);
  }
  if (tid == 0) A.tau[r] = tau;
}

__global__ void __launch_bounds__(kTopkThreads, 1) select_kernel(const FusedSelArgs A) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  const int r = blockIdx.x, tid = threadIdx.x;
  int* out = A.idx + static_cast<long long>(r) * A.k;
  const long long n = row_pos(A, r) + 1;
  if (n <= A.k) {
    for (int j = tid; j < A.k; j += kTopkThreads) out[j] = j < n ? j : -1;
    return;
  }
  const unsigned cnt = A.cand_count[r];
  if (cnt < static_cast<unsigned>(A.k) || cnt > static_cast<unsigned>(A.cand_cap) ||
      A.cand_cap > kCandCap || n > kSampledMaxN) {
    if (tid == 0) {
      A.fail_rows[atomicAdd(A.fail_count, 1u)] = r;
      atomicAdd(A.fail_total, 1u);
    }
    return;
  }
  const unsigned* ck = A.cand_key + static_cast<long long>(r) * A.cand_cap;
  const int* ci = A.cand_idx + static_cast<long long>(r) * A.cand_cap;
  for (unsigned j = tid; j < cnt; j += kTopkThreads) {
    sm.cand_key[j] = ck[j];
    sm.cand_idx[j] = ci[j];
  }
  __syncthreads();
  select_from_candidates(n, A.k, static_cast<int>(cnt), out, sm);
}

__device__ __forceinline__ float e4m3_float(uint8_t c) {
  __nv_fp8_e4m3 v;
  v.__x = c;
  return static_cast<float>(v);
}

// One listed row per CTA at a time: its scores over keys 0 .. pos, the same
// formula as the indexer (the dot product of the e4m3 codes in fp32, ReLU,
// the folded weight w * scale * q_scale, the sum over heads, then k_scale),
// into this CTA's scratch row; then the full top-k of that row. The sums run
// in another order than the tensor cores' and the indexer epilogue's, so a
// recomputed score equals the indexer's exactly only where every partial sum
// is exact (the integer FP8 grid), and otherwise to within fp32 rounding.
template <int HI>
__global__ void __launch_bounds__(kTopkThreads, 1) fallback_kernel(const FusedSelArgs A) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  float* qf = reinterpret_cast<float*>(smem_raw + ((sizeof(TopkSmem) + 15) / 16) * 16);
  float* wq = qf + HI * 128;
  const int tid = threadIdx.x;
  const unsigned nfail = *A.fail_count;
  float* sc = A.scratch + static_cast<long long>(blockIdx.x) * A.ld;
  for (unsigned f = blockIdx.x; f < nfail; f += gridDim.x) {
    const int r = A.fail_rows[f];
    const long long n = row_pos(A, r) + 1;
    __syncthreads();
    for (int j = tid; j < HI * 128; j += kTopkThreads)
      qf[j] = e4m3_float(A.q8[static_cast<long long>(r) * HI * 128 + j]);
    for (int h = tid; h < HI; h += kTopkThreads)
      wq[h] = A.w[static_cast<long long>(r) * HI + h] *
              (A.scale * (A.q_scale ? A.q_scale[r] : 1.f));
    __syncthreads();
    for (long long s = tid; s < n; s += kTopkThreads) {
      float acc[HI];
#pragma unroll
      for (int h = 0; h < HI; ++h) acc[h] = 0.f;
      const uint4* kr = reinterpret_cast<const uint4*>(A.k8 + s * 128);
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        const uint4 u = kr[c];
        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
        float kf[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) kf[j] = e4m3_float(static_cast<uint8_t>(wd[j >> 2] >> (8 * (j & 3))));
#pragma unroll
        for (int h = 0; h < HI; ++h) {
          const float* qh = qf + h * 128 + 16 * c;
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[h] = fmaf(qh[j], kf[j], acc[h]);
        }
      }
      float I = 0.f;
#pragma unroll
      for (int h = 0; h < HI; ++h) I = fmaf(wq[h], fmaxf(acc[h], 0.f), I);
      sc[s] = I * (A.k_scale ? A.k_scale[s] : 1.f);
    }
    __syncthreads();
    select_row(sc, n, A.k, A.idx + static_cast<long long>(r) * A.k, sm);
  }
}

size_t topk_smem() { return sizeof(TopkSmem); }

template <typename K>
cudaError_t prepare(K kern, size_t smem) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  return e;
}

template <int HI>
cudaError_t launch_fallback_hi(const FusedSelArgs& a, cudaStream_t st) {
  const size_t smem = (topk_smem() + 15) / 16 * 16 + sizeof(float) * (HI * 128 + HI);
  cudaError_t e = prepare(fallback_kernel<HI>, smem);
  if (e != cudaSuccess) return e;
  fallback_kernel<HI><<<a.slots, kTopkThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fused_tau(const FusedSelArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  cudaError_t e = prepare(tau_kernel, topk_smem());
  if (e != cudaSuccess) return e;
  tau_kernel<<<a.T, kTopkThreads, topk_smem(), st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fused_select(const FusedSelArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  cudaError_t e = prepare(select_kernel, topk_smem());
  if (e != cudaSuccess) return e;
  select_kernel<<<a.T, kTopkThreads, topk_smem(), st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fused_fallback(const FusedSelArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  switch (a.Hi) {
    case 1: return launch_fallback_hi<1>(a, st);
    case 2: return launch_fallback_hi<2>(a, st);
    case 4: return launch_fallback_hi<4>(a, st);
    case 8: return launch_fallback_hi<8>(a, st);
    case 16: return launch_fallback_hi<16>(a, st);
    case 32: return launch_fallback_hi<32>(a, st);
    case 64: return launch_fallback_hi<64>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsa

// warmup.cu -- the indexer's warm-up objective, forward and backward, sm_100a.
//
// "ele-yufo.com/posts/deepseek-v3-2-exp", section "四、训练的两步走冷启动":
// before sparse training, dense attention is run and the weight distribution
// each token receives is recorded as the target; with the main model frozen,
// the lightning indexer alone is trained with a KL divergence to fit it.
// Readings: the target of query t is the dense causal attention distribution
// averaged over the heads, p[t,s] = (1/H) sum_h softmax_s(sm_scale q[t,h].kv[s]);
// the indexer's distribution is r[t,s] = softmax_s(I[t,s]) over the same
// causal keys; the loss of row t is KL(p_t || r_t) and its gradient with
// respect to the scores is r - p. The backward continues through the indexer
// I = sum_h w * ReLU(scale * qf . kf) to the dequantised inputs qf, kf and w;
// the ReLU's decision is taken on the raw FP8 dot product, as in the forward.
//
// The attention logits of the target come from the tcgen05 GEMM; the rest are
// plain CUDA-core kernels in fp32 (one CTA per query row, or per block of
// keys): the objective is a training-time step, measured but not tuned like
// the inference path.
#include "common.cuh"
#include "dsa_internal.h"
#include <cuda_fp8.h>

namespace dsa {
namespace {

constexpr int kWThreads = 256;

__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < kWThreads / 32; ++w) t += red[w];
  return t;
}

__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = -INFINITY;
  for (int w = 0; w < kWThreads / 32; ++w) t = fmaxf(t, red[w]);
  return t;
}

__device__ __forceinline__ float e4m3_value(uint8_t c) {
  __nv_fp8_e4m3 v;
  v.__x = c;
  return static_cast<float>(v);
}

// p[t][s] = mean over heads of the dense causal attention weights, from the
// logits z[t*H + h][s] = q[t,h] . kv[s] (the tensor-core GEMM) and the per-head
// log normaliser lse[t][h] (natural log, as dsa_sparse_mla_fwd returns it for
// index sets covering the prefix). Keys past the row's position get 0.
__global__ void __launch_bounds__(kWThreads) probs_kernel(const float* __restrict__ z,
                                                          long long ldz,
                                                          const float* __restrict__ lse, int S,
                                                          int H, int q_pos0, float sm_scale,
                                                          float* __restrict__ p, long long ldp) {
  __shared__ float ls[128];
  const long long t = blockIdx.x;
  const long long pos = min(static_cast<long long>(q_pos0) + t, static_cast<long long>(S) - 1);
  for (int h = threadIdx.x; h < H; h += kWThreads) ls[h] = lse[t * H + h];
  __syncthreads();
  const float inv_h = 1.f / H;
  const float* zr = z + t * H * ldz;
  for (long long s = threadIdx.x; s < S; s += kWThreads) {
    float acc = 0.f;
    if (s <= pos)
      for (int h = 0; h < H; ++h) acc += expf(sm_scale * zr[h * ldz + s] - ls[h]);
    p[t * ldp + s] = acc * inv_h;
  }
}

// loss[t] = KL(p_t || softmax(I_t)) over the causal keys; grad[t][s] = r - p
// (0 past the row's keys).
__global__ void __launch_bounds__(kWThreads) kl_kernel(const float* __restrict__ I, long long ldi,
                                                       const float* __restrict__ p, long long ldp,
                                                       int S, int q_pos0, float* __restrict__ loss,
                                                       float* __restrict__ grad, long long ldg) {
  __shared__ float red[kWThreads / 32];
  const long long t = blockIdx.x;
  const long long n = min(static_cast<long long>(q_pos0) + t + 1, static_cast<long long>(S));
  const float* ir = I + t * ldi;
  const float* pr = p + t * ldp;
  float m = -INFINITY;
  for (long long s = threadIdx.x; s < n; s += kWThreads) m = fmaxf(m, ir[s]);
  m = block_max(m, red);
  float z = 0.f;
  for (long long s = threadIdx.x; s < n; s += kWThreads) z += expf(ir[s] - m);
  z = block_sum(z, red);
  const float logz = m + logf(z);
  float kl = 0.f;
  float* gr = grad + t * ldg;
  for (long long s = threadIdx.x; s < S; s += kWThreads) {
    float g = 0.f;
    if (s < n) {
      const float lr = ir[s] - logz, ps = pr[s];
      if (ps > 0.f) kl += ps * (logf(ps) - lr);
      g = expf(lr) - ps;
    }
    gr[s] = g;
  }
  kl = block_sum(kl, red);
  if (threadIdx.x == 0) loss[t] = kl;
}

constexpr int kQKeys = 32;     // keys per block in the per-query kernel
constexpr int kKKeys = 16;     // keys per CTA in the per-key kernel

// The ReLU's decision is taken on the raw e4m3 dot product xr = q8 . k8 (the
// scales are positive), as the forward indexer takes it; the scales enter the
// magnitudes only: x = q_scale * k_scale * xr.
//
// Per query t, over its keys in blocks of 32:
//   dq[t,h,:] = w[t,h] scale sum_s g[t,s] [xr > 0] k_scale[s] k8[s,:]
//   dw[t,h]   = sum_s g[t,s] scale q_scale[t] k_scale[s] max(xr, 0)
__global__ void __launch_bounds__(kWThreads) bwd_query_kernel(const IndexerBwdArgs A) {
  extern __shared__ float smem[];
  const int Hi = A.Hi;
  float* qr = smem;                          // [Hi][128] e4m3 values
  float* kr = qr + Hi * 128;                 // [32][128] e4m3 values
  float* xs = kr + kQKeys * 128;             // [32][Hi] raw dot products
  float* gs = xs + kQKeys * Hi;              // [32] g * k_scale
  const long long t = blockIdx.x;
  const long long n = min(static_cast<long long>(A.q_pos0) + t + 1, static_cast<long long>(A.S));
  const float qsc = A.q_scale ? A.q_scale[t] : 1.f;
  for (int j = threadIdx.x; j < Hi * 128; j += kWThreads) qr[j] = e4m3_value(A.q8[t * Hi * 128 + j]);
  constexpr int kOut = 32;                   // outputs per thread: Hi * 128 / 256 <= 32
  float acc[kOut];
#pragma unroll
  for (int i = 0; i < kOut; ++i) acc[i] = 0.f;
  float dw = 0.f;
  const float* g = A.grad + t * A.ldg;
  for (long long s0 = 0; s0 < n; s0 += kQKeys) {
    __syncthreads();
    for (int j = threadIdx.x; j < kQKeys * 128; j += kWThreads) {
      const long long s = s0 + j / 128;
      kr[j] = s < n ? e4m3_value(A.k8[s * 128 + (j % 128)]) : 0.f;
    }
    if (threadIdx.x < kQKeys) {
      const long long s = s0 + threadIdx.x;
      gs[threadIdx.x] = s < n ? g[s] * (A.k_scale ? A.k_scale[s] : 1.f) : 0.f;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < kQKeys * Hi; j += kWThreads) {
      const int ks = j / Hi, h = j % Hi;
      float x = 0.f;
      for (int d = 0; d < 128; ++d) x = fmaf(qr[h * 128 + d], kr[ks * 128 + d], x);
      xs[ks * Hi + h] = x;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kOut; ++i) {
      const int o = threadIdx.x + kWThreads * i;
      if (o < Hi * 128) {
        const int h = o / 128, d = o % 128;
        float a = acc[i];
        for (int ks = 0; ks < kQKeys; ++ks)
          if (xs[ks * Hi + h] > 0.f) a = fmaf(gs[ks], kr[ks * 128 + d], a);
        acc[i] = a;
      }
    }
    if (threadIdx.x < Hi)
      for (int ks = 0; ks < kQKeys; ++ks)
        dw = fmaf(gs[ks], fmaxf(xs[ks * Hi + threadIdx.x], 0.f), dw);
  }
#pragma unroll
  for (int i = 0; i < kOut; ++i) {
    const int o = threadIdx.x + kWThreads * i;
    if (o < Hi * 128) A.dq[t * Hi * 128 + o] = acc[i] * A.w[t * Hi + o / 128] * A.scale;
  }
  if (threadIdx.x < Hi) A.dw[t * Hi + threadIdx.x] = dw * A.scale * qsc;
}

// Per block of 16 keys, over the queries that see them:
//   dk[s,:] = scale sum_t sum_h g[t,s] w[t,h] [xr > 0] q_scale[t] q8[t,h,:]
__global__ void __launch_bounds__(kWThreads) bwd_key_kernel(const IndexerBwdArgs A) {
  extern __shared__ float smem[];
  const int Hi = A.Hi;
  float* kr = smem;                          // [16][128] e4m3 values
  float* qr = kr + kKKeys * 128;             // [Hi][128] e4m3 values of query t
  float* xs = qr + Hi * 128;                 // [16][Hi] coefficients
  float* gs = xs + kKKeys * Hi;              // [16]
  float* ws = gs + kKKeys;                   // [Hi]
  const long long s0 = static_cast<long long>(blockIdx.x) * kKKeys;
  for (int j = threadIdx.x; j < kKKeys * 128; j += kWThreads) {
    const long long s = s0 + j / 128;
    kr[j] = s < A.S ? e4m3_value(A.k8[s * 128 + (j % 128)]) : 0.f;
  }
  constexpr int kOut = kKKeys * 128 / kWThreads;   // 8
  float acc[kOut];
#pragma unroll
  for (int i = 0; i < kOut; ++i) acc[i] = 0.f;
  // queries that see key s0 (position q_pos0 + t >= s0)
  const long long t0 = max(0ll, s0 - A.q_pos0);
  for (long long t = t0; t < A.T; ++t) {
    __syncthreads();
    for (int j = threadIdx.x; j < Hi * 128; j += kWThreads) qr[j] = e4m3_value(A.q8[t * Hi * 128 + j]);
    const long long pos = static_cast<long long>(A.q_pos0) + t;
    const float qsc = A.q_scale ? A.q_scale[t] : 1.f;
    if (threadIdx.x < kKKeys) {
      const long long s = s0 + threadIdx.x;
      gs[threadIdx.x] = (s < A.S && s <= pos) ? A.grad[t * A.ldg + s] * qsc : 0.f;
    }
    for (int h = threadIdx.x; h < Hi; h += kWThreads) ws[h] = A.w[t * Hi + h];
    __syncthreads();
    for (int j = threadIdx.x; j < kKKeys * Hi; j += kWThreads) {
      const int ks = j / Hi, h = j % Hi;
      float x = 0.f;
      for (int d = 0; d < 128; ++d) x = fmaf(qr[h * 128 + d], kr[ks * 128 + d], x);
      xs[ks * Hi + h] = x > 0.f ? gs[ks] * ws[h] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kOut; ++i) {
      const int o = threadIdx.x + kWThreads * i;   // (key, dim) = (o / 128, o % 128)
      const int ks = o / 128, d = o % 128;
      float a = acc[i];
      for (int h = 0; h < Hi; ++h) a = fmaf(xs[ks * Hi + h], qr[h * 128 + d], a);
      acc[i] = a;
    }
  }
#pragma unroll
  for (int i = 0; i < kOut; ++i) {
    const int o = threadIdx.x + kWThreads * i;
    const long long s = s0 + o / 128;
    if (s < A.S) A.dk[s * 128 + (o % 128)] = acc[i] * A.scale;
  }
}

}  // namespace

cudaError_t launch_attention_probs(const void* q, const void* kv, const float* lse, int T, int S,
                                   int H, int q_pos0, float sm_scale, float* p, long long ldp,
                                   float* z, long long ldz, unsigned* err, cudaStream_t st) {
  cudaError_t e = launch_gemm_f32(q, kv, z, T * H, S, 576, ldz, err, st);
  if (e != cudaSuccess) return e;
  probs_kernel<<<T, kWThreads, 0, st>>>(z, ldz, lse, S, H, q_pos0, sm_scale, p, ldp);
  return cudaGetLastError();
}

cudaError_t launch_indexer_kl(const float* I, long long ldi, const float* p, long long ldp, int T,
                              int S, int q_pos0, float* loss, float* grad, long long ldg,
                              cudaStream_t st) {
  kl_kernel<<<T, kWThreads, 0, st>>>(I, ldi, p, ldp, S, q_pos0, loss, grad, ldg);
  return cudaGetLastError();
}

cudaError_t launch_indexer_backward(const IndexerBwdArgs& a, cudaStream_t st) {
  const size_t sq = sizeof(float) * (a.Hi * 128 + kQKeys * 128 + kQKeys * a.Hi + kQKeys);
  const size_t sk = sizeof(float) * (kKKeys * 128 + a.Hi * 128 + kKKeys * a.Hi + kKKeys + a.Hi);
  cudaError_t e = cudaFuncSetAttribute(bwd_query_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sq));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(bwd_key_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sk));
  if (e != cudaSuccess) return e;
  bwd_query_kernel<<<a.T, kWThreads, sq, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_key_kernel<<<(a.S + kKKeys - 1) / kKKeys, kWThreads, sk, st>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa

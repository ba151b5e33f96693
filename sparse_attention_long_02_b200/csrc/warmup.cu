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
// The attention logits of the target and the three products of the backward
// are tcgen05 GEMMs; the reductions and coefficients around them are
// CUDA-core kernels in fp32 over coalesced rows.
#include "common.cuh"
#include "dsa_internal.h"
#include <cuda_fp8.h>
#include <cuda_bf16.h>
#include <algorithm>

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

// The ReLU's decision is taken on the raw e4m3 dot product xr = q8 . k8 (the
// scales are positive), as the forward indexer takes it; the scales enter the
// magnitudes only: x = q_scale * k_scale * xr. With r = (t, h) a row of the
// T*Hi query heads and pos(t) = min(q_pos0 + t, S - 1):
//   dq[r,:] = sum_s Cq[r,s] k8[s,:],  Cq[r,s] = [s <= pos(t)][xr > 0] g[t,s] k_scale[s] w[r] scale
//   dk[s,:] = sum_r Ck[s,r] q8[r,:],  Ck[s,r] = [s <= pos(t)][xr > 0] g[t,s] q_scale[t] w[r] scale
//   dw[r]   = scale q_scale[t] sum_{s <= pos(t)} g[t,s] k_scale[s] max(xr, 0)
// xr, dq and dk are tcgen05 GEMMs. The e4m3 codes are exact in bf16, and each
// fp32 coefficient is written as three bf16 pieces whose sum is exactly that
// coefficient (8 + 8 + 8 significant bits); the pieces lie side by side along
// K against the same B, so every product in the tensor core is exact and the
// accumulation is fp32.

__device__ __forceinline__ void split3(float v, __nv_bfloat16& a, __nv_bfloat16& b,
                                       __nv_bfloat16& c) {
  a = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(a);      // exact: at most 16 significant bits
  b = __float2bfloat16_rn(r1);
  c = __float2bfloat16_rn(r1 - __bfloat162float(b));
}

__device__ __forceinline__ uint2 pack4(__nv_bfloat16 a, __nv_bfloat16 b, __nv_bfloat16 c,
                                       __nv_bfloat16 d) {
  uint2 u;
  u.x = static_cast<uint32_t>(__bfloat16_as_ushort(a)) |
        (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
  u.y = static_cast<uint32_t>(__bfloat16_as_ushort(c)) |
        (static_cast<uint32_t>(__bfloat16_as_ushort(d)) << 16);
  return u;
}

// Writes the three pieces of four consecutive coefficients v[0..3] at column c
// of a row whose pieces start every `piece` elements.
__device__ __forceinline__ void store_split4(__nv_bfloat16* row, long long piece, long long c,
                                             const float (&v)[4]) {
  __nv_bfloat16 p[3][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) split3(v[j], p[0][j], p[1][j], p[2][j]);
#pragma unroll
  for (int k = 0; k < 3; ++k)
    *reinterpret_cast<uint2*>(row + k * piece + c) = pack4(p[k][0], p[k][1], p[k][2], p[k][3]);
}

// e4m3 rows [rows][128] -> bf16 copies: dst [rows][128] and its transpose
// dstT [128][ldT] (columns rows .. ldT - 1 zero). One CTA per 64 rows.
__global__ void __launch_bounds__(kWThreads) to_bf16_kernel(const uint8_t* __restrict__ src,
                                                            long long rows,
                                                            __nv_bfloat16* __restrict__ dst,
                                                            __nv_bfloat16* __restrict__ dstT,
                                                            long long ldT) {
  __shared__ float tile[64][129];
  const long long r0 = static_cast<long long>(blockIdx.x) * 64;
  for (int j = threadIdx.x; j < 64 * 128; j += kWThreads) {
    const int i = j / 128, d = j % 128;
    const long long r = r0 + i;
    const float v = r < rows ? e4m3_value(src[r * 128 + d]) : 0.f;
    tile[i][d] = v;
    if (r < rows) dst[r * 128 + d] = __float2bfloat16_rn(v);
  }
  __syncthreads();
  for (int j = threadIdx.x; j < 64 * 128; j += kWThreads) {
    const int d = j / 64, i = j % 64;
    dstT[d * ldT + r0 + i] = __float2bfloat16_rn(tile[i][d]);
  }
}

// One CTA per query-head row r: the pieces of Cq[r, 0 .. Sp) and dw[r].
__global__ void __launch_bounds__(kWThreads) coef_q_kernel(const IndexerBwdArgs A,
                                                           const float* __restrict__ x,
                                                           long long ldx,
                                                           __nv_bfloat16* __restrict__ cq,
                                                           long long Sp) {
  __shared__ float red[kWThreads / 32];
  const long long r = blockIdx.x, t = r / A.Hi;
  const long long pos = min(static_cast<long long>(A.q_pos0) + t, static_cast<long long>(A.S) - 1);
  const float wsc = A.w[r] * A.scale;
  const float* xr = x + r * ldx;
  const float* g = A.grad + t * A.ldg;
  __nv_bfloat16* row = cq + r * 3 * Sp;
  float dw = 0.f;
  for (long long s = 4ll * threadIdx.x; s < Sp; s += 4 * kWThreads) {
    float4 x4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (s < A.S) x4 = *reinterpret_cast<const float4*>(xr + s);   // s + 3 < ldx
    const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
    float v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[j] = 0.f;
      if (s + j <= pos) {
        const float gk = g[s + j] * (A.k_scale ? A.k_scale[s + j] : 1.f);
        if (xv[j] > 0.f) {
          v[j] = gk * wsc;
          dw = fmaf(gk, xv[j], dw);
        }
      }
    }
    store_split4(row, Sp, s, v);
  }
  dw = block_sum(dw, red);
  if (threadIdx.x == 0) A.dw[r] = dw * A.scale * (A.q_scale ? A.q_scale[t] : 1.f);
}

// Grid (S, column blocks of 1024): the pieces of Ck[s, 0 .. Kp) for key s,
// from xt = xr transposed ([S][ldxt]).
__global__ void __launch_bounds__(kWThreads) coef_k_kernel(const IndexerBwdArgs A,
                                                           const float* __restrict__ xt,
                                                           long long ldxt,
                                                           __nv_bfloat16* __restrict__ ck,
                                                           long long Kp) {
  const long long s = blockIdx.x;
  const long long c = 4 * (static_cast<long long>(blockIdx.y) * kWThreads + threadIdx.x);
  if (c >= Kp) return;
  const long long R = static_cast<long long>(A.T) * A.Hi;
  float4 x4 = make_float4(0.f, 0.f, 0.f, 0.f);
  if (c < R) x4 = *reinterpret_cast<const float4*>(xt + s * ldxt + c);   // c + 3 < ldxt
  const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
  float v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[j] = 0.f;
    const long long r = c + j, t = r / A.Hi;
    if (r < R && A.q_pos0 + t >= s && xv[j] > 0.f)
      v[j] = A.grad[t * A.ldg + s] * (A.q_scale ? A.q_scale[t] : 1.f) * A.w[r] * A.scale;
  }
  store_split4(ck + s * 3 * Kp, Kp, c, v);
}

// dk = sum over the splits of the split-K partial products.
__global__ void __launch_bounds__(kWThreads) sum_splits_kernel(const float* __restrict__ part,
                                                               int splits, long long n,
                                                               float* __restrict__ out) {
  const long long i = static_cast<long long>(blockIdx.x) * kWThreads + threadIdx.x;
  if (i >= n) return;
  float a = 0.f;
  for (int z = 0; z < splits; ++z) a += part[z * n + i];
  out[i] = a;
}

long long round_to(long long v, long long m) { return (v + m - 1) / m * m; }

// Workspace of the backward, each part 256-byte aligned.
struct BwdLayout {
  long long R, Sp, Kp, ldx, ldxt;
  int splits, kps;
  size_t x, c, qb, qbt, kb, kbt, part, total;
};

BwdLayout bwd_layout(int T, int S, int Hi) {
  BwdLayout L;
  L.R = static_cast<long long>(T) * Hi;
  L.Sp = round_to(S, 64);
  L.Kp = round_to(L.R, 64);
  L.ldx = round_to(S, 4);
  L.ldxt = round_to(L.R, 4);
  // dk: S / 128 row tiles of one 128-column tile; split K to fill the 148 SMs
  const int m_tiles = (S + 127) / 128;
  const int nk = static_cast<int>(3 * L.Kp / 64);
  L.splits = std::max(1, std::min(nk, 148 / m_tiles));
  L.kps = (nk + L.splits - 1) / L.splits;
  L.splits = (nk + L.kps - 1) / L.kps;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  };
  L.x = take(4 * static_cast<size_t>(std::max(L.R * L.ldx, static_cast<long long>(S) * L.ldxt)));
  L.c = take(2 * static_cast<size_t>(std::max(L.R * 3 * L.Sp, static_cast<long long>(S) * 3 * L.Kp)));
  L.qb = take(2 * static_cast<size_t>(L.R) * 128);
  L.qbt = take(2 * static_cast<size_t>(L.Kp) * 128);
  L.kb = take(2 * static_cast<size_t>(S) * 128);
  L.kbt = take(2 * static_cast<size_t>(L.Sp) * 128);
  L.part = take(4 * static_cast<size_t>(L.splits) * S * 128);
  L.total = off;
  return L;
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

size_t indexer_backward_workspace(int T, int S, int Hi) { return bwd_layout(T, S, Hi).total; }

cudaError_t launch_indexer_backward(const IndexerBwdArgs& a, void* workspace, unsigned* err,
                                    cudaStream_t st) {
  const BwdLayout L = bwd_layout(a.T, a.S, a.Hi);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* x = reinterpret_cast<float*>(ws + L.x);
  __nv_bfloat16* c = reinterpret_cast<__nv_bfloat16*>(ws + L.c);
  __nv_bfloat16* qb = reinterpret_cast<__nv_bfloat16*>(ws + L.qb);
  __nv_bfloat16* qbt = reinterpret_cast<__nv_bfloat16*>(ws + L.qbt);
  __nv_bfloat16* kb = reinterpret_cast<__nv_bfloat16*>(ws + L.kb);
  __nv_bfloat16* kbt = reinterpret_cast<__nv_bfloat16*>(ws + L.kbt);
  float* part = reinterpret_cast<float*>(ws + L.part);
  const int R = static_cast<int>(L.R);
  to_bf16_kernel<<<static_cast<unsigned>(L.Kp / 64), kWThreads, 0, st>>>(a.q8, L.R, qb, qbt, L.Kp);
  to_bf16_kernel<<<static_cast<unsigned>(L.Sp / 64), kWThreads, 0, st>>>(a.k8, a.S, kb, kbt, L.Sp);
  cudaError_t e = cudaGetLastError();
  // xr [R][S] -> Cq, dw -> dq
  if (e == cudaSuccess) e = launch_gemm_f32(qb, kb, x, R, a.S, 128, L.ldx, err, st);
  if (e != cudaSuccess) return e;
  coef_q_kernel<<<R, kWThreads, 0, st>>>(a, x, L.ldx, c, L.Sp);
  e = cudaGetLastError();
  if (e == cudaSuccess)
    e = launch_gemm_f32(c, kbt, a.dq, R, 128, static_cast<int>(3 * L.Sp), 128, err, st,
                        static_cast<int>(L.Sp));
  // xr transposed [S][R] -> Ck -> dk (split K, then the sum of the splits)
  if (e == cudaSuccess) e = launch_gemm_f32(kb, qb, x, a.S, R, 128, L.ldxt, err, st);
  if (e != cudaSuccess) return e;
  coef_k_kernel<<<dim3(a.S, static_cast<unsigned>((L.Kp / 4 + kWThreads - 1) / kWThreads)),
                  kWThreads, 0, st>>>(a, x, L.ldxt, c, L.Kp);
  e = cudaGetLastError();
  if (e == cudaSuccess)
    e = launch_gemm_f32(c, qbt, part, a.S, 128, static_cast<int>(3 * L.Kp), 128, err, st,
                        static_cast<int>(L.Kp), L.kps);
  if (e != cudaSuccess) return e;
  const long long n = static_cast<long long>(a.S) * 128;
  sum_splits_kernel<<<static_cast<unsigned>((n + kWThreads - 1) / kWThreads), kWThreads, 0, st>>>(
      part, L.splits, n, a.dk);
  return cudaGetLastError();
}

}  // namespace dsa

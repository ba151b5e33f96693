// proj.cu -- projection of hidden states to the FP8 indexer inputs, sm_100a.
//
// Step 1 of the four-step workflow ("DeepSeek-V3.2-Exp 模型优势与 DSA 工作原理",
// section 4 "步骤一：查询与键的投影"; "devpress.csdn.net ... DSA", section
// "第一步：查询与键的投影"): the hidden states H are projected to queries
// Q = H W_Q and keys K = H W_K, rotary position encoding is applied to both,
// and each head gets a weight a_h, a further linear map of H. The indexer
// reads Q and K as FP8 with one fp32 scale per token.
//
// Kernel 1, a tcgen05 GEMM: Y = H W^T for W = [W_Q | W_K | W_a] stored as
// [N][d] rows (N = Hi*128 + 128 + Hi), one 128-token x 256-output tile per
// CTA, K in 64-wide steps through a four-stage TMA ring. The epilogue rotates
// each (2i, 2i+1) pair of the q and k columns by the caller's cos/sin table
// at the token's position, writes q and k in fp32 to the workspace with each
// token's |y| maximum (one atomic per tile and part), and writes a_h.
// Kernel 2 quantises q and k per token: scale = amax / 448 (1 if amax = 0),
// code = e4m3(y / scale), rounded to nearest even and saturated at +-448.
//
// The same GEMM with a plain epilogue (every output written in fp32) serves
// the indexer's warm-up objective: the attention logits of its target, and
// the products of its backward. For those, B's K coordinate may wrap (A holds
// several K-blocks that all multiply the same B), and a launch may split K
// over grid.z, split z writing its partial product at y + z * M * ldy.
#include "common.cuh"
#include "dsa_internal.h"
#include <cuda_fp8.h>

namespace dsa {
namespace {

constexpr int kProjThreads = 256;        // warp 0 TMA, warp 1 MMA, warps 4-7 epilogue
constexpr int kBM = 128, kBN = 256, kBK = 64, kPStages = 4;
constexpr int kATile = kBM * kBK * 2;    // 128 tokens x 64 dims bf16
constexpr int kBTile = kBN * kBK * 2;    // 256 outputs x 64 dims bf16

struct ProjSmem {
  uint8_t a[kPStages][kATile];
  uint8_t b[kPStages][kBTile];
  unsigned long long full[kPStages];
  unsigned long long empty[kPStages];
  unsigned long long done;
  uint32_t tmem_base;
  int abort_flag;
};

template <bool kPlain>
__global__ void __launch_bounds__(kProjThreads, 1)
proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                 const ProjArgs P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  ProjSmem& sm = *reinterpret_cast<ProjSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned* err = P.err;
  if (launch_aborted(err)) return;
  const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * kBM;
  // K steps of this CTA: all of them, or split z of a split-K launch
  const int nk_all = (P.d + kBK - 1) / kBK;
  const int per = P.kt_split > 0 ? P.kt_split : nk_all;
  const int kt0 = blockIdx.z * per;
  const int nk = min(per, nk_all - kt0);
  const int kbw = P.kb > 0 ? P.kb : P.d;          // B's K extent: its coordinate wraps
  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(smem_u32(&sm.full[i]), 1);
      mbar_init(smem_u32(&sm.empty[i]), 1);
    }
    mbar_init(smem_u32(&sm.done), 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int st = i % kPStages;
        if (i >= kPStages &&
            !mbar_wait(smem_u32(&sm.empty[st]), ((i / kPStages) + 1) & 1, abort_flag, err))
          break;
        const uint32_t full = smem_u32(&sm.full[st]);
        const int k = (kt0 + i) * kBK;
        mbar_expect_tx(full, kATile + kBTile);
        tma_load_2d(smem_u32(sm.a[st]), &tm_h, full, k, m0);
        tma_load_2d(smem_u32(sm.b[st]), &tm_w, full, k % kbw, n0);
        ++issued;
      }
      for (int i = issued > kPStages ? issued - kPStages : 0; i < issued; ++i)
        mbar_drain(smem_u32(&sm.full[i % kPStages]), (i / kPStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kBM, kBN, false);
      for (int kt = 0; kt < nk; ++kt) {
        const int st = kt % kPStages;
        if (!mbar_wait(smem_u32(&sm.full[st]), (kt / kPStages) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint64_t ad = sdesc_sw128(smem_u32(sm.a[st]), 0, 1024);
        const uint64_t bd = sdesc_sw128(smem_u32(sm.b[st]), 0, 1024);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)     // K = 16 per MMA (32 bytes)
          mma_bf16(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
        mma_commit(smem_u32(&sm.empty[st]));
      }
      mma_commit(smem_u32(&sm.done));
      mbar_drain(smem_u32(&sm.done), 0);
    }
  } else if (warp >= 4) {
    // --------------------------------------------------------- epilogue
    const int row = 32 * (warp & 3) + lane;       // TMEM lane = token of the tile
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const long long t = static_cast<long long>(m0) + row;
    const int nq = P.Hi * 128, nqk = nq + 128;
    if (warp_wait(smem_u32(&sm.done), 0, abort_flag, err)) {
      tc_fence_after();
      float amax_q = 0.f, amax_k = 0.f;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        const int col0 = n0 + 32 * c;
        float y[32];
        tmem_ld32(tmem + lane_base + 32 * c, y);
        if (t >= P.T || col0 >= P.N) continue;
        if constexpr (kPlain) {
          float* dst = P.y + blockIdx.z * P.zstride + t * P.ldy + col0;
          if (col0 + 32 <= P.N) {        // rows and y 16-byte aligned (ldy % 4 == 0)
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(dst + j) = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < P.N) dst[j] = y[j];
          }
          continue;
        }
        if (col0 < nqk) {
          // q or k columns: rotate the 16 pairs of this chunk by the token's table
          const float2* cs = reinterpret_cast<const float2*>(P.rope) + t * 64 + (col0 % 128) / 2;
          float m = 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float2 r = cs[j];
            const float u = y[2 * j], v = y[2 * j + 1];
            y[2 * j] = u * r.x - v * r.y;
            y[2 * j + 1] = u * r.y + v * r.x;
            m = fmaxf(m, fmaxf(fabsf(y[2 * j]), fabsf(y[2 * j + 1])));
          }
          if (col0 < nq) amax_q = fmaxf(amax_q, m);
          else amax_k = fmaxf(amax_k, m);
          float4* dst = reinterpret_cast<float4*>(P.y + t * nqk + col0);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(y[4 * e], y[4 * e + 1], y[4 * e + 2], y[4 * e + 3]);
        } else {
          // per-head weights a_h (columns past N are padding)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < P.N) P.a[t * P.Hi + (col0 + j - nqk)] = y[j];
        }
      }
      // bit patterns of non-negative floats order like the floats
      if (!kPlain && t < P.T && amax_q > 0.f) atomicMax(P.amax_q + t, __float_as_uint(amax_q));
      if (!kPlain && t < P.T && amax_k > 0.f) atomicMax(P.amax_k + t, __float_as_uint(amax_k));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBN);
  }
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE,
                                                           __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE,
                                                           __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// One CTA per token: per-token scales and e4m3 codes of q and k.
__global__ void __launch_bounds__(256) proj_quant_kernel(const ProjArgs P) {
  const long long t = blockIdx.x;
  const int nq = P.Hi * 128, nqk = nq + 128;
  const float aq = __uint_as_float(P.amax_q[t]), ak = __uint_as_float(P.amax_k[t]);
  const float sq = aq > 0.f ? aq / 448.f : 1.f;
  const float sk = ak > 0.f ? ak / 448.f : 1.f;
  if (threadIdx.x == 0) {
    P.q_scale[t] = sq;
    P.k_scale[t] = sk;
  }
  const float4* yr = reinterpret_cast<const float4*>(P.y + t * nqk);
  uint32_t* q8 = reinterpret_cast<uint32_t*>(P.q8 + t * nq);
  uint32_t* k8 = reinterpret_cast<uint32_t*>(P.k8 + t * 128);
  for (int j4 = threadIdx.x; j4 < nqk / 4; j4 += blockDim.x) {
    const float4 v = yr[j4];
    const bool isq = 4 * j4 < nq;
    const float s = isq ? sq : sk;
    const uint32_t packed = e4m3x4(v.x / s, v.y / s, v.z / s, v.w / s);
    if (isq) q8[j4] = packed;
    else k8[j4 - nq / 4] = packed;
  }
}

}  // namespace

template <bool kPlain>
cudaError_t launch_gemm(const ProjArgs& a, const void* h, const void* wt, cudaStream_t st) {
  CUtensorMap th, tw;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cudaError_t e = make_tmap_2d(&th, h, bf, a.d, a.T, static_cast<uint64_t>(a.d) * 2, kBK, kBM,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  const int kbw = a.kb > 0 ? a.kb : a.d;
  if (e == cudaSuccess)
    e = make_tmap_2d(&tw, wt, bf, kbw, a.N, static_cast<uint64_t>(kbw) * 2, kBK, kBN,
                     CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(ProjSmem) + 1024;
  e = cudaFuncSetAttribute(proj_gemm_kernel<kPlain>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int nk = (a.d + kBK - 1) / kBK;
  const int splits = a.kt_split > 0 ? (nk + a.kt_split - 1) / a.kt_split : 1;
  dim3 grid((a.N + kBN - 1) / kBN, (a.T + kBM - 1) / kBM, splits);
  proj_gemm_kernel<kPlain><<<grid, kProjThreads, smem, st>>>(th, tw, a);
  return cudaGetLastError();
}

cudaError_t launch_project(const ProjArgs& a, const void* h, const void* wt, cudaStream_t st) {
  cudaError_t e = launch_gemm<false>(a, h, wt, st);
  if (e != cudaSuccess) return e;
  proj_quant_kernel<<<a.T, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gemm_f32(const void* a, const void* b, float* c, int M, int N, int K,
                            long long ldc, unsigned* err, cudaStream_t st, int kb, int kt_split) {
  ProjArgs P;
  P.T = M;
  P.N = N;
  P.d = K;
  P.kb = kb;
  P.kt_split = kt_split;
  P.y = c;
  P.ldy = ldc;
  P.zstride = static_cast<long long>(M) * ldc;
  P.err = err;
  return launch_gemm<true>(P, a, b, st);
}

}  // namespace dsa

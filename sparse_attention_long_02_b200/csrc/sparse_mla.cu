// sparse_mla.cu -- sparse MLA attention over the selected latent rows, sm_100a.
//
// Step 4 of the four-step workflow ("DeepSeek-V3.2-Exp 模型优势与 DSA 工作原理",
// section 4): attention is computed only over the positions the top-k
// selected, the softmax is normalised within those positions, and the output
// is the weighted sum of the selected values. The keys are the 512-d latent
// rows (page 3, section 3 "稀疏多潜在注意力"), here 512 latent + 64 rope
// dims, and the values are the same rows' 512 latent dims; all heads of a
// query share one gathered row, so the head x key contraction runs on the
// tensor cores.
//
// Layout of the work. One query (all H <= 128 heads on the MMA's M) runs on a
// cluster of two CTAs. A 128-head x 512-dim fp32 output needs all 512 TMEM
// columns of an SM, so the output is split by value dims: CTA 0 owns latent
// dims [0,256) and CTA 1 owns [256,512). The logit contraction is split the
// same way, CTA 0 also taking the 64 rope dims, so each CTA gathers only the
// dims it uses and every selected byte crosses HBM once. Per tile of 64
// selected keys:
//   1. warp 0 gathers the CTA's dims of the 64 rows with TMA gather4 (the
//      block table is applied here for the paged cache);
//   2. warp 1 issues S_c = Q_c K_c^T (M=128 heads, N=64 keys) into TMEM;
//   3. warps 4-7 (one thread per head) read their partial logits, push them
//      to the peer CTA's shared memory, add the peer's partials (fp32 adds
//      commute, so both CTAs see identical logits), run the online softmax
//      in the exp2 domain and write P (bf16) for the tensor core; the
//      running maximum is re-based only when it grows by more than 8 (log2
//      units), and only then is the TMEM output rescaled;
//   4. warp 1 issues O_c += P V_c (M=128, N=256 dims, K=64 keys), reading V
//      from the same gathered tile (MN-major view).
// The final output is O / l in bf16 and lse = (m + log2 l) * ln 2.
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kMlaThreads = 256;
constexpr int kTileKeys = 64;
constexpr int kStages = 2;
constexpr int kAtomBytesQ = 128 * 128;          // 128 heads x 64 dims bf16
constexpr int kAtomBytesKV = kTileKeys * 128;   // 64 keys x 64 dims bf16
constexpr int kMaxAtoms = 5;
constexpr uint32_t kColO = 0;                   // TMEM columns [0,256): output
constexpr uint32_t kColS = 256;                 // [256,384): two logit buffers
constexpr float kRebase = 8.0f;                 // lazy rescale threshold (log2 units)

struct MlaSmem {
  uint8_t q[kMaxAtoms][kAtomBytesQ];
  uint8_t kv[kStages][kMaxAtoms][kAtomBytesKV];
  uint8_t p[128 * 128];                         // P: 128 heads x 64 keys bf16, SW128
  float x[128 * 64];                            // peer's partial logits (swizzled rows)
  unsigned long long q_full;
  unsigned long long kv_full[kStages];
  unsigned long long kv_empty[kStages];
  unsigned long long s_full[2];
  unsigned long long s_empty[2];
  unsigned long long p_full;
  unsigned long long p_empty;
  unsigned long long x_full;                    // peer wrote into x
  unsigned long long x_free;                    // peer finished reading its own x
  unsigned long long o_done;
  uint32_t tmem_base;
  int abort_flag;
};

// 64-dim atom a of this CTA -> first dim of the atom in the 576-dim row.
__device__ __forceinline__ int atom_dim(int rank, int a) {
  return rank == 0 ? (a < 4 ? 64 * a : 512) : 256 + 64 * a;
}

// Physical row of selected slot `v` (a logical position), or -1 if skipped.
__device__ __forceinline__ int kv_row(const MlaArgs& A, int v, int seq, int limit) {
  if (v < 0) return -1;
  if (v >= limit) {
    raise_error(A.err, kErrBounds);
    return -1;
  }
  if (!A.block_table) return v;
  const int pb = A.block_table[static_cast<long long>(seq) * A.max_blocks + (v >> 6)];
  if (pb < 0 || pb >= A.nblk) {
    raise_error(A.err, kErrBounds);
    return -1;
  }
  return pb * 64 + (v & 63);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMlaThreads, 1)
sparse_mla_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                  const MlaArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  MlaSmem& sm = *reinterpret_cast<MlaSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned* err = A.err;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const int nat = rank == 0 ? 5 : 4;
  const int r = blockIdx.x >> 1;                 // query row (one cluster per row)
  const int seq = A.block_table ? r / A.nq : 0;
  // keys a slot may name: the causal prefix of the query (paged) or the cache
  int limit = A.S;
  if (A.block_table) limit = A.seq_len[seq] - A.nq + (r % A.nq) + 1;
  const int ntiles = (A.k + kTileKeys - 1) / kTileKeys;
  const int* sel = A.idx + static_cast<long long>(r) * A.k;
  const int warp = warp_id(), lane = lane_id();
  // Both CTAs of the pair take the same early exit, so neither waits alone.
  const bool aborted = launch_aborted(err);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.q_full), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&sm.kv_full[i]), 1);
      mbar_init(smem_u32(&sm.kv_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.s_empty[i]), 128);
    }
    mbar_init(smem_u32(&sm.p_full), 128);
    mbar_init(smem_u32(&sm.p_empty), 1);
    mbar_init(smem_u32(&sm.x_full), 128);
    mbar_init(smem_u32(&sm.x_free), 128);
    mbar_init(smem_u32(&sm.o_done), 1);
    sm.abort_flag = aborted ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();          // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0 && !aborted) {
    // ------------------------------------------------------- gather warp
    if (lane == 0) {
      mbar_expect_tx(smem_u32(&sm.q_full), nat * kAtomBytesQ);
      for (int a = 0; a < nat; ++a)
        tma_load_2d(smem_u32(sm.q[a]), &tm_q, smem_u32(&sm.q_full), atom_dim(rank, a), r * A.H);
    }
    int issued = 0;
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % kStages;
      if (i >= kStages &&
          !warp_wait(smem_u32(&sm.kv_empty[st]), ((i / kStages) + 1) & 1, abort_flag, err))
        break;
      const uint32_t full = smem_u32(&sm.kv_full[st]);
      if (lane == 0) mbar_expect_tx(full, nat * kAtomBytesKV);
      __syncwarp();
      if (lane < 16) {
        int rows[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int j = i * kTileKeys + 4 * lane + c;
          const int v = j < A.k ? sel[j] : -1;
          const int pr = kv_row(A, v, seq, limit);
          rows[c] = pr < 0 ? A.kv_rows : pr;     // past the end: TMA fills zeros
        }
        for (int a = 0; a < nat; ++a)
          tma_gather4(smem_u32(sm.kv[st][a]) + lane * 512, &tm_kv, full, atom_dim(rank, a),
                      rows[0], rows[1], rows[2], rows[3]);
      }
      ++issued;
    }
    if (lane == 0) {
      for (int i = max(0, issued - kStages); i < issued; ++i)
        mbar_drain(smem_u32(&sm.kv_full[i % kStages]), (i / kStages) & 1);
      mbar_drain(smem_u32(&sm.q_full), 0);
    }
  } else if (warp == 1 && !aborted) {
    // ------------------------------------------------------- MMA thread
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(128, kTileKeys, false);
      const uint32_t id_pv = idesc_bf16(128, 256, true);
      const uint64_t pdesc = sdesc_sw128(smem_u32(sm.p), 0, 1024);
      bool ok = mbar_wait(smem_u32(&sm.q_full), 0, abort_flag, err);
      auto issue_pv = [&](int i) -> bool {
        const int st = i % kStages;
        if (!mbar_wait(smem_u32(&sm.p_full), i & 1, abort_flag, err)) return false;
        tc_fence_after();
        const uint64_t vdesc = sdesc_sw128(smem_u32(sm.kv[st][0]), kAtomBytesKV, 1024);
#pragma unroll
        for (int kk = 0; kk < kTileKeys / 16; ++kk)   // 16 keys = 2 groups of 8 rows
          mma_bf16(tmem + kColO, pdesc + 2 * kk, vdesc + (kk * 2048 >> 4), id_pv,
                   (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(smem_u32(&sm.p_empty));
        mma_commit(smem_u32(&sm.kv_empty[st]));
        return true;
      };
      int done_pv = 0;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int st = i % kStages, b = i & 1;
        if (!mbar_wait(smem_u32(&sm.kv_full[st]), (i / kStages) & 1, abort_flag, err)) break;
        if (i >= 2 && !mbar_wait(smem_u32(&sm.s_empty[b]), ((i >> 1) + 1) & 1, abort_flag, err))
          break;
        tc_fence_after();
        for (int a = 0; a < nat; ++a) {
          const uint64_t qd = sdesc_sw128(smem_u32(sm.q[a]), 0, 1024);
          const uint64_t kd = sdesc_sw128(smem_u32(sm.kv[st][a]), 0, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)          // 4 x K=16 dims (32 bytes)
            mma_bf16(tmem + kColS + b * kTileKeys, qd + 2 * kk, kd + 2 * kk, id_qk,
                     (a > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(smem_u32(&sm.s_full[b]));
        if (i > 0) {
          if (!issue_pv(i - 1)) break;
          done_pv = i;
        }
      }
      if (ok && done_pv == ntiles - 1 && !*abort_flag) issue_pv(ntiles - 1);
      mma_commit(smem_u32(&sm.o_done));
      mbar_drain(smem_u32(&sm.o_done), 0);
    }
  } else if (warp >= 4 && !aborted) {
    // ------------------------------------------------- softmax warpgroup
    const int h = 32 * (warp & 3) + lane;               // head = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t peer_x = mapa(smem_u32(sm.x), peer) + h * 256;
    const uint32_t peer_x_full = mapa(smem_u32(&sm.x_full), peer);
    const uint32_t peer_x_free = mapa(smem_u32(&sm.x_free), peer);
    const float* my_x = sm.x + h * 64;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; ok && i < ntiles; ++i) {
      const int b = i & 1;
      float s[64];
      if (!(ok = warp_wait(smem_u32(&sm.s_full[b]), (i >> 1) & 1, abort_flag, err))) break;
      tc_fence_after();
      tmem_ld32(tmem + lane_base + kColS + b * kTileKeys, *reinterpret_cast<float(*)[32]>(s));
      tmem_ld32(tmem + lane_base + kColS + b * kTileKeys + 32,
                *reinterpret_cast<float(*)[32]>(s + 32));
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.s_empty[b]));
      // exchange partial logits with the peer CTA
      if (i > 0 && !(ok = warp_wait<true>(smem_u32(&sm.x_free), (i - 1) & 1, abort_flag, err)))
        break;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int pc = c ^ (h & 7);
        st_cluster_v4(peer_x + pc * 16, s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
      }
      mbar_arrive_remote(peer_x_full);
      if (!(ok = warp_wait<true>(smem_u32(&sm.x_full), i & 1, abort_flag, err))) break;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int pc = c ^ (h & 7);
        const float4 v = *reinterpret_cast<const float4*>(my_x + pc * 4);
        s[4 * c] += v.x;
        s[4 * c + 1] += v.y;
        s[4 * c + 2] += v.z;
        s[4 * c + 3] += v.w;
      }
      mbar_arrive_remote(peer_x_free);
      // mask unselected slots, scale into the log2 domain
      float mt = -INFINITY;
      const int* tsel = sel + i * kTileKeys;
#pragma unroll
      for (int c = 0; c < kTileKeys; c += 4) {
        int4 v4 = make_int4(-1, -1, -1, -1);
        if (i * kTileKeys + c + 3 < A.k) v4 = __ldg(reinterpret_cast<const int4*>(tsel + c));
        else {
          int* pv = reinterpret_cast<int*>(&v4);
          for (int e = 0; e < 4; ++e)
            if (i * kTileKeys + c + e < A.k) pv[e] = __ldg(tsel + c + e);
        }
        const int vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool valid = vv[e] >= 0 && vv[e] < limit;
          s[c + e] = valid ? s[c + e] * A.sm_scale_log2 : -INFINITY;
          mt = fmaxf(mt, s[c + e]);
        }
      }
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_ref + kRebase) {        // also the first tile with a valid key
        const float m_new = fmaxf(mt, m_ref);
        if (m_ref > -INFINITY) {
          alpha = exp2f(m_ref - m_new);
          rescale = true;
        }
        m_ref = m_new;
      }
      float psum = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = m_ref > -INFINITY ? exp2f(s[2 * c] - m_ref) : 0.f;
        const float p1 = m_ref > -INFINITY ? exp2f(s[2 * c + 1] - m_ref) : 0.f;
        psum += p0 + p1;
        const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
        pk[c] = *reinterpret_cast<const uint32_t*>(&pb);
      }
      l = l * alpha + psum;
      // P buffer and the output are free once PV(i-1) has finished
      if (i > 0 && !(ok = warp_wait(smem_u32(&sm.p_empty), (i - 1) & 1, abort_flag, err))) break;
      if (rescale && i > 0) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          float o[32];
          tmem_ld32(tmem + lane_base + kColO + 32 * c, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tmem + lane_base + kColO + 32 * c, o);
        }
      }
      // P row h: 64 bf16 = 128 B in the 128-B swizzle (chunk c at c ^ (h % 8))
      uint8_t* prow = sm.p + (h >> 3) * 1024 + (h & 7) * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int pc = c ^ (h & 7);
        *reinterpret_cast<uint4*>(prow + pc * 16) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.p_full));
    }
    // ------------------------------------------------------- epilogue
    if (ok && ntiles > 0 &&
        warp_wait(smem_u32(&sm.p_empty), (ntiles - 1) & 1, abort_flag, err)) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const bool head_ok = h < A.H;
      __nv_bfloat16* orow = A.out + (static_cast<long long>(r) * A.H + h) * 512 + rank * 256;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_base + kColO + 32 * c, o);
        if (head_ok) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
            pk[e] = *reinterpret_cast<const uint32_t*>(&v);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (rank == 0 && head_ok && A.lse)
        A.lse[static_cast<long long>(r) * A.H + h] =
            l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();          // the peer no longer touches this CTA's shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_sparse_mla(const MlaArgs& a_in, const void* q, const void* kv, long long kv_rows,
                              long long q_rows, cudaStream_t st) {
  MlaArgs a = a_in;
  a.kv_rows = static_cast<int>(kv_rows);
  CUtensorMap tq, tkv;
  cudaError_t e = make_tmap_2d(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 576, q_rows, 576 * 2, 64,
                               128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&tkv, kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 576, kv_rows, 576 * 2, 64, 1,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(MlaSmem) + 1024;
  e = cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(2 * a.T);      // x has no 65535 limit; cluster pairs are consecutive x
  sparse_mla_kernel<<<grid, kMlaThreads, smem, st>>>(tq, tkv, a);
  return cudaGetLastError();
}

size_t sparse_mla_smem_bytes() { return sizeof(MlaSmem) + 1024; }

}  // namespace dsa

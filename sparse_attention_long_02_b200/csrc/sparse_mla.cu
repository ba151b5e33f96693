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
// columns of an SM, so the output is split by value dims: CTA c owns latent
// dims [256c, 256c+256). The logit contraction is split the same way, each
// CTA also taking half of the 64 rope dims ([512+32c, 512+32c+32)), so both
// CTAs do the same work, each gathers only the dims it uses, and every
// selected byte crosses HBM once. Per tile of 64 selected keys:
//   1. six gather warps copy the CTA's dims of the 64 rows with coalesced
//      cp.async (through the block table for the paged cache), up to four
//      tiles ahead;
//   2. warp 1 issues S_c = Q_c K_c^T (M=128 heads, N=64 keys, K=288) with
//      Q_c read from TMEM, where it was placed once per query, and K_c from
//      the gathered tile, into the TMEM logit buffer;
//   3. eight softmax warps, two per TMEM lane quarter (thread = head, each
//      warp of a pair taking 32 of the 64 keys), scale their partial logits
//      into the log2 domain and stage them, in fp32, in shared memory; the
//      exchange warp sends the whole 32 KB tile to the peer CTA with one bulk
//      copy (the TMA engine, off the load/store path the gather uses). Tile
//      i+1 is staged and sent while tile i is finished, so the transfer runs
//      under the softmax arithmetic. Both CTAs add the same two fp32
//      partials (fp32 addition commutes), so they see identical logits with
//      nothing rounded below fp32; they mask unselected slots, agree on
//      the tile maximum through shared memory, run the online softmax in the
//      exp2 domain and store P (bf16) into the TMEM P buffer; the
//      running maximum is re-based only when it grows by more than 8 (log2
//      units), and only then is the output in TMEM rescaled;
//   4. warp 1 issues O_c += P V_c with P read from TMEM (M=128, N=256 dims,
//      K=64 keys) and V from the same gathered tile (MN-major view).
// The final output is O / l in bf16 and lse = (m + log2 l) * ln 2.
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kMlaThreads = 512;
constexpr int kTileKeys = 64;
constexpr int kStages = 3;
constexpr int kAtoms = 4;                        // 128-B swizzled atoms of 64 dims
constexpr int kAtomBytesQ = 128 * 128;           // 128 heads x 64 dims bf16
constexpr int kRopeBytesQ = 128 * 64;            // 128 heads x 32 dims bf16 (64-B swizzle)
constexpr int kAtomBytesKV = kTileKeys * 128;    // 64 keys x 64 dims bf16
constexpr int kRopeBytesKV = kTileKeys * 64;     // 64 keys x 32 dims bf16
constexpr int kGatherWarps = 6;                  // warps 0, 2, 3, 12, 13, 14
constexpr int kSoftmaxWarps = 8;                 // warps 4-11
constexpr int kExchangeWarp = 15;
constexpr uint32_t kXBytes = 128 * kTileKeys * 4;   // one tile of fp32 partial logits
constexpr uint32_t kColO = 0;                    // TMEM columns [0,256): output
constexpr uint32_t kColQ = 256;                  // [256,400): Q_c, bf16 pairs (256 + 32 dims)
constexpr uint32_t kColP = 416;                  // [416,448): P, bf16 pairs
constexpr uint32_t kColS = 448;                  // [448,512): logits
// Q arrives by TMA in the exchange buffers (latent atoms 0-1 in x, 2-3 in
// stage[0], the rope block in stage[1]) and is moved into TMEM before the
// first exchange, so the whole KV ring is free for the gather from the first
// tile.
constexpr float kRebase = 8.0f;                  // lazy rescale threshold (log2 units)

// Rows of 64 fp32 partials (256 B, one per head); the 16-B chunk c of row h
// sits at chunk c ^ (h & 7), so eight consecutive heads hit distinct banks.
struct MlaSmem {
  uint8_t kv[kStages][kAtoms][kAtomBytesKV];
  uint8_t kv_rope[kStages][kRopeBytesKV];
  uint4 x[128 * 16];                             // the peer's partials of the current tile
  uint4 stage[2][128 * 16];                      // this CTA's partials (bulk copy source), by tile parity
  float pair_max[2][2][128];                     // [tile parity][key half][head]
  unsigned valid[kStages][2];                    // selected-slot bits of each half tile
  unsigned long long q_full;                     // Q has landed in its staging slots
  unsigned long long q_ready;                    // Q is in TMEM (its staging slots are free)
  unsigned long long peer_q;                     // the peer's Q is in its TMEM: its x may be sent to
  unsigned long long kv_full[kStages];
  unsigned long long kv_empty[kStages];
  unsigned long long s_full;
  unsigned long long s_empty;
  unsigned long long p_full;
  unsigned long long p_empty;
  // per send buffer (tile parity):
  unsigned long long stage_full[2];              // the eight softmax warps have staged a tile
  unsigned long long stage_free[2];              // the peer has received the tile staged here
  unsigned long long x_full;                     // the peer's partials have landed in x
  unsigned long long x_free;                     // the peer has read what this CTA sent it
  unsigned long long x_read;                     // the softmax warps have read x
  unsigned long long pair;                       // the softmax warps have posted their maxima
  unsigned long long o_done;
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(MlaSmem::x) == 2 * kAtomBytesQ, "two Q atoms per exchange buffer");
static_assert(sizeof(MlaSmem::stage[0]) == 2 * kAtomBytesQ, "two Q atoms per exchange buffer");
static_assert(sizeof(MlaSmem::stage[1]) >= kRopeBytesQ, "Q rope block fits a stage buffer");
static_assert(kAtomBytesKV % 1024 == 0 && kRopeBytesKV % 1024 == 0, "1024-B aligned staging");

// Shared-memory address of Q staging atom a (0-3): atoms 0-1 in x, 2-3 in
// stage[0]; and the generic pointer of a shared-memory address of `sm`.
__device__ __forceinline__ uint32_t q_atom(MlaSmem& sm, int a) {
  return (a < 2 ? smem_u32(sm.x) : smem_u32(sm.stage[0])) + (a & 1) * kAtomBytesQ;
}
__device__ __forceinline__ const uint8_t* smem_generic(MlaSmem& sm, uint32_t saddr) {
  return reinterpret_cast<const uint8_t*>(&sm) + (saddr - smem_u32(&sm));
}

// Physical block of slot value `v` (a logical position) in the paged cache,
// loaded a tile ahead of its use; -1 when no lookup is needed.
__device__ __forceinline__ int kv_block(const MlaArgs& A, int v, int seq, int limit) {
  if (!A.block_table || v < 0 || v >= limit) return -1;
  return __ldg(A.block_table + static_cast<long long>(seq) * A.max_blocks + (v >> 6));
}

// Physical row of slot value `v` given its block `pb` (kv_block), or -1 if
// the slot is skipped.
__device__ __forceinline__ int kv_row(const MlaArgs& A, int v, int pb, int limit) {
  if (v < 0) return -1;
  if (v >= limit) {
    raise_error(A.err, kErrBounds);
    return -1;
  }
  if (!A.block_table) return v;
  if (pb < 0 || pb >= A.nblk) {
    raise_error(A.err, kErrBounds);
    return -1;
  }
  return pb * 64 + (v & 63);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMlaThreads, 1)
sparse_mla_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                  const MlaArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  MlaSmem& sm = *reinterpret_cast<MlaSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned* err = A.err;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const int r = blockIdx.x >> 1;                 // query row (one cluster per row)
  const int seq = A.block_table ? r / A.nq : 0;
  // keys a slot may name: the causal prefix of the query (paged) or the cache
  int limit = A.S;
  if (A.block_table) limit = A.seq_len[seq] - A.nq + (r % A.nq) + 1;
  const int ntiles = (A.k + kTileKeys - 1) / kTileKeys;
  const int* sel = A.idx + static_cast<long long>(r) * A.k;
  const int warp = warp_id(), lane = lane_id();
  const int dim0 = 256 * static_cast<int>(rank);             // first latent dim of this CTA
  const int rope0 = 512 + 32 * static_cast<int>(rank);       // first rope dim of this CTA
  // Both CTAs of the pair normally take the same early exit; if they did not,
  // the working one times out on the peer's barriers and still returns.
  const bool aborted = launch_aborted(err);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_ready), 4);         // the four warps that move Q into TMEM
    mbar_init(smem_u32(&sm.peer_q), 1);          // one arrival from the peer
    for (int i = 0; i < kStages; ++i) {
      // one cp.async-completion arrival per gathering thread + the slot writer
      mbar_init(smem_u32(&sm.kv_full[i]), 32 * kGatherWarps + 1);
      mbar_init(smem_u32(&sm.kv_empty[i]), 1);
    }
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.s_empty), kSoftmaxWarps);
    mbar_init(smem_u32(&sm.p_full), kSoftmaxWarps);
    mbar_init(smem_u32(&sm.p_empty), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.stage_full[b]), kSoftmaxWarps);
      mbar_init(smem_u32(&sm.stage_free[b]), 1);  // one arrival from the peer per use
    }
    mbar_init(smem_u32(&sm.x_full), 1);          // own expect_tx + the peer's copied bytes
    mbar_init(smem_u32(&sm.x_free), 1);          // one arrival from the peer per use
    mbar_init(smem_u32(&sm.x_read), kSoftmaxWarps);
    mbar_init(smem_u32(&sm.pair), kSoftmaxWarps);
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

  const bool gather = warp == 0 || warp == 2 || warp == 3 || (warp >= 12 && warp <= 14);
  if (gather && !aborted) {
    // ------------------------------------------------------- gather warps
    // Each warp copies whole rows: one cp.async per lane covers the 512-B latent
    // slice of a row (coalesced), lanes 0-3 add its 64-B rope slice; rows land
    // in the 128-B (latent) and 64-B (rope) swizzled layouts the MMA reads.
    const int gw = warp == 0 ? 0 : warp <= 3 ? warp - 1 : warp - 9;   // 0..5
    if (warp == 0 && lane == 0) {
      const uint32_t qf = smem_u32(&sm.q_full);
      mbar_expect_tx(qf, kAtoms * kAtomBytesQ + kRopeBytesQ);
      for (int a = 0; a < kAtoms; ++a)
        tma_load_2d(q_atom(sm, a), &tm_q, qf, dim0 + 64 * a, r * A.H);
      tma_load_2d(smem_u32(sm.stage[1]), &tm_qr, qf, rope0, r * A.H);
    }
    // Two-deep prefetch: the slots of tile i+2 and the block-table entries
    // of tile i+1 are loading while tile i is issued.
    auto slot = [&](int j) { return j < A.k ? __ldg(sel + j) : -1; };
    int v0 = slot(lane), v1 = slot(lane + 32);                          // tile 0
    int b0 = kv_block(A, v0, seq, limit), b1 = kv_block(A, v1, seq, limit);
    int n0 = slot(kTileKeys + lane), n1 = slot(kTileKeys + lane + 32);  // tile 1
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % kStages;
      const int c0 = v0, c1 = v1, p0 = b0, p1 = b1;
      if (i + 1 < ntiles) {
        v0 = n0;
        v1 = n1;
        b0 = kv_block(A, v0, seq, limit);
        b1 = kv_block(A, v1, seq, limit);
      }
      if (i + 2 < ntiles) {
        n0 = slot((i + 2) * kTileKeys + lane);
        n1 = slot((i + 2) * kTileKeys + lane + 32);
      }
      const int r0 = kv_row(A, c0, p0, limit), r1 = kv_row(A, c1, p1, limit);
      if (i >= kStages &&
          !warp_wait(smem_u32(&sm.kv_empty[st]), ((i / kStages) + 1) & 1, abort_flag, err))
        break;
      const uint32_t full = smem_u32(&sm.kv_full[st]);
      if (gw == 0) {
        const unsigned b0 = __ballot_sync(0xffffffffu, r0 >= 0);
        const unsigned b1 = __ballot_sync(0xffffffffu, r1 >= 0);
        if (lane == 0) {
          sm.valid[st][0] = b0;
          sm.valid[st][1] = b1;
          mbar_arrive(full);
        }
      }
      const uint32_t kv0 = smem_u32(sm.kv[st][lane >> 3]);
      const uint32_t rope = smem_u32(sm.kv_rope[st]);
      for (int row = gw; row < kTileKeys; row += kGatherWarps) {
        const int pr = __shfl_sync(0xffffffffu, row < 32 ? r0 : r1, row & 31);
        const __nv_bfloat16* src = A.kv + static_cast<long long>(pr < 0 ? 0 : pr) * 576;
        const uint32_t nb = pr < 0 ? 0u : 16u;               // skipped slot: zero fill
        cp_async16(kv0 + row * 128 + (((lane & 7) ^ (row & 7)) << 4), src + dim0 + lane * 8, nb);
        if (lane < 4)
          cp_async16(rope + row * 64 + ((lane ^ ((row >> 1) & 3)) << 4), src + rope0 + lane * 8, nb);
      }
      cp_async_arrive(full);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (warp == 0 && lane == 0) mbar_drain(smem_u32(&sm.q_full), 0);
  } else if (warp == kExchangeWarp && !aborted) {
    // ---------------------------------------------------- exchange warp
    // Tile j's partials travel from stage[j & 1] to the peer's x in one bulk
    // copy, once they are staged and the peer has read tile j-1 out of x
    // (for tile 0: once the peer has moved its Q, which is staged in x, into
    // TMEM). The send side is double-buffered, so staging tile j+1 never
    // waits for tile j's copy; the receive side is single, so the copy of
    // tile j+1 starts once both CTAs have read tile j, while both finish it.
    // This warp also tells the peer when its copy of tile i has landed here
    // (that stage buffer may be refilled) and when x has been read (it may
    // send the next tile). Cluster-scope releases come from this warp only,
    // so they never queue behind the softmax warps.
    if (lane == 0) {
      int sent = 0;
      auto send = [&](int j) -> bool {
        const int b = j & 1;
        if (!mbar_wait(smem_u32(&sm.stage_full[b]), (j >> 1) & 1, abort_flag, err)) return false;
        if (j >= 1 && !mbar_wait<true>(smem_u32(&sm.x_free), (j - 1) & 1, abort_flag, err))
          return false;
        bulk_copy_to_peer(mapa(smem_u32(sm.x), peer), smem_u32(sm.stage[b]), kXBytes,
                          mapa(smem_u32(&sm.x_full), peer));
        sent = j + 1;
        return true;
      };
      if (ntiles > 0) mbar_expect_tx(smem_u32(&sm.x_full), kXBytes);        // the peer's tile 0
      // this CTA's Q has left x: the peer may send into it
      bool ok = mbar_wait(smem_u32(&sm.q_ready), 0, abort_flag, err);
      if (ok) mbar_arrive_remote(mapa(smem_u32(&sm.peer_q), peer));
      ok = ok && mbar_wait<true>(smem_u32(&sm.peer_q), 0, abort_flag, err);
      ok = ok && (ntiles == 0 || send(0));
      for (int i = 0; ok && i < ntiles; ++i) {
        if (!(ok = mbar_wait<true>(smem_u32(&sm.x_full), i & 1, abort_flag, err))) break;
        mbar_arrive_remote(mapa(smem_u32(&sm.stage_free[i & 1]), peer));
        if (!(ok = mbar_wait(smem_u32(&sm.x_read), i & 1, abort_flag, err))) break;
        // armed before the peer may send tile i+1 (it waits for x_free)
        if (i + 1 < ntiles) mbar_expect_tx(smem_u32(&sm.x_full), kXBytes);
        mbar_arrive_remote(mapa(smem_u32(&sm.x_free), peer));
        if (i + 1 < ntiles && !(ok = send(i + 1))) break;
      }
      // A copy reads this CTA's stage buffer until it lands: wait for the
      // peer's word on the last two before this CTA may leave (the softmax
      // warps waited for every earlier one before restaging).
      for (int j = sent > 2 ? sent - 2 : 0; j < sent; ++j) {
        const uint32_t bar = smem_u32(&sm.stage_free[j & 1]);
        if (!mbar_wait<true>(bar, (j >> 1) & 1, abort_flag, err)) mbar_drain(bar, (j >> 1) & 1);
      }
    }
  } else if (warp == 1 && !aborted) {
    // ------------------------------------------------------- MMA thread
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(128, kTileKeys, false);
      const uint32_t id_pv = idesc_bf16(128, 256, true);
      bool ok = mbar_wait(smem_u32(&sm.q_ready), 0, abort_flag, err);
      // debug: o_done completes only after the commit below, so this bounded
      // wait runs out and both CTAs leave through their give-up paths
      if (ok && (debug_bits(err) & kDbgStallMla))
        ok = mbar_wait(smem_u32(&sm.o_done), 0, abort_flag, err);
      auto issue_pv = [&](int i) -> bool {
        const int st = i % kStages;
        if (!mbar_wait(smem_u32(&sm.p_full), i & 1, abort_flag, err)) return false;
        tc_fence_after();
        const uint64_t vdesc = sdesc_sw128(smem_u32(sm.kv[st][0]), kAtomBytesKV, 1024);
#pragma unroll
        for (int kk = 0; kk < kTileKeys / 16; ++kk)   // 16 keys: 8 P columns, 2 V row groups
          mma_bf16_ts(tmem + kColO, tmem + kColP + 8 * kk, vdesc + (kk * 2048 >> 4), id_pv,
                      (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(smem_u32(&sm.p_empty));
        mma_commit(smem_u32(&sm.kv_empty[st]));
        return true;
      };
      // QK runs two tiles ahead of PV: the softmax reads tile i+1's logits
      // while it finishes tile i
      int next_pv = 0;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int st = i % kStages;
        if (!mbar_wait(smem_u32(&sm.kv_full[st]), (i / kStages) & 1, abort_flag, err)) break;
        // the softmax warps have read the previous tile's logits
        if (i >= 1 && !mbar_wait(smem_u32(&sm.s_empty), (i - 1) & 1, abort_flag, err)) break;
        fence_proxy_async_smem();         // cp.async (generic) writes -> tensor-core reads
        tc_fence_after();
        const uint32_t d = tmem + kColS;
        for (int a = 0; a < kAtoms; ++a) {
          const uint64_t kd = sdesc_sw128(smem_u32(sm.kv[st][a]), 0, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)          // 4 x K=16 dims (8 TMEM columns of Q)
            mma_bf16_ts(d, tmem + kColQ + 32 * a + 8 * kk, kd + 2 * kk, id_qk,
                        (a > 0 || kk > 0) ? 1u : 0u);
        }
        {
          const uint64_t kd = sdesc_sw64(smem_u32(sm.kv_rope[st]), 512);
          mma_bf16_ts(d, tmem + kColQ + 128, kd, id_qk, 1u);
          mma_bf16_ts(d, tmem + kColQ + 136, kd + 2, id_qk, 1u);
        }
        mma_commit(smem_u32(&sm.s_full));
        if (i >= 2) {
          if (!(ok = issue_pv(i - 2))) break;
          next_pv = i - 1;
        }
      }
      while (ok && next_pv < ntiles && !*abort_flag && issue_pv(next_pv)) ++next_pv;
      mma_commit(smem_u32(&sm.o_done));
      mbar_drain(smem_u32(&sm.o_done), 0);
    }
  } else if (warp >= 4 && warp < 4 + kSoftmaxWarps && !aborted) {
    // ------------------------------------------------- softmax warps
    const int g = (warp - 4) >> 2;                      // key half of the tile
    const int h = 32 * (warp & 3) + lane;               // head = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    if (g == 0) {
      // Move this head's row of Q_c from its staging slots into TMEM (bf16
      // pairs, lane = head): 256 latent dims from the 128-B swizzled atoms,
      // then the 32 rope dims from the 64-B swizzled block.
      if ((ok = warp_wait(smem_u32(&sm.q_full), 0, abort_flag, err))) {
#pragma unroll 1
        for (int a = 0; a < kAtoms; ++a) {
          const uint4* row = reinterpret_cast<const uint4*>(smem_generic(sm, q_atom(sm, a)) + h * 128);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 v = row[(4 * half + c) ^ (h & 7)];
              pk[4 * c] = v.x;
              pk[4 * c + 1] = v.y;
              pk[4 * c + 2] = v.z;
              pk[4 * c + 3] = v.w;
            }
            tmem_st16(tmem + lane_base + kColQ + 32 * a + 16 * half, pk);
          }
        }
        {
          const uint4* row = reinterpret_cast<const uint4*>(
              reinterpret_cast<const uint8_t*>(sm.stage[1]) + h * 64);
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = row[c ^ ((h >> 1) & 3)];
            pk[4 * c] = v.x;
            pk[4 * c + 1] = v.y;
            pk[4 * c + 2] = v.z;
            pk[4 * c + 3] = v.w;
          }
          tmem_st16(tmem + lane_base + kColQ + 128, pk);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.q_ready));
      }
    }
    // This warp's half of tile j's partial logits, scaled into log2 units
    // (fp32), staged for the peer in stage[j & 1] once the copy of tile j-2
    // out of that buffer has landed.
    auto stage_tile = [&](int j) -> bool {
      const int b = j & 1;
      float v32[32];
      if (!warp_wait(smem_u32(&sm.s_full), j & 1, abort_flag, err)) return false;
      tc_fence_after();
      tmem_ld32(tmem + lane_base + kColS + 32 * g, v32);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.s_empty));
      if (j >= 2 &&
          !warp_wait<true>(smem_u32(&sm.stage_free[b]), ((j - 2) >> 1) & 1, abort_flag, err))
        return false;
      uint4* dst = sm.stage[b] + h * 16;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        dst[(8 * g + c) ^ (h & 7)] =
            make_uint4(__float_as_uint(v32[4 * c] * A.sm_scale_log2),
                       __float_as_uint(v32[4 * c + 1] * A.sm_scale_log2),
                       __float_as_uint(v32[4 * c + 2] * A.sm_scale_log2),
                       __float_as_uint(v32[4 * c + 3] * A.sm_scale_log2));
      fence_proxy_async_smem();           // generic writes -> the bulk copy's reads
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.stage_full[b]));
      return true;
    };
    if (ok && ntiles > 0) ok = stage_tile(0);
    for (int i = 0; ok && i < ntiles; ++i) {
      const int st = i % kStages, b = i & 1;
      // which slots of this half tile are selected (staged by the gather warp)
      if (!(ok = warp_wait(smem_u32(&sm.kv_full[st]), (i / kStages) & 1, abort_flag, err))) break;
      const unsigned valid = sm.valid[st][g];
      // own + peer partials, then hand x back
      if (!(ok = warp_wait<true>(smem_u32(&sm.x_full), i & 1, abort_flag, err))) break;
      float s[32];
      {
        const uint4* xp = sm.x + h * 16;
        const uint4* op = sm.stage[b] + h * 16;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 f = xp[(8 * g + c) ^ (h & 7)];
          const uint4 o = op[(8 * g + c) ^ (h & 7)];
          s[4 * c] = __uint_as_float(o.x) + __uint_as_float(f.x);
          s[4 * c + 1] = __uint_as_float(o.y) + __uint_as_float(f.y);
          s[4 * c + 2] = __uint_as_float(o.z) + __uint_as_float(f.z);
          s[4 * c + 3] = __uint_as_float(o.w) + __uint_as_float(f.w);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.x_read));
      // the next tile's partials go out while this one is finished
      if (i + 1 < ntiles && !(ok = stage_tile(i + 1))) break;
      if (valid != 0xffffffffu) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (!((valid >> j) & 1u)) s[j] = -INFINITY;
      }
      float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 32; ++j) pm[j & 3] = fmaxf(pm[j & 3], s[j]);
      const float my_max = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
      // the tile maximum of this head: both halves post theirs
      sm.pair_max[i & 1][g][h] = my_max;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.pair));
      if (!(ok = warp_wait(smem_u32(&sm.pair), i & 1, abort_flag, err))) break;
      const float mt = fmaxf(my_max, sm.pair_max[i & 1][g ^ 1][h]);
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_ref + kRebase) {        // also the first tile with a selected key
        if (m_ref > -INFINITY) {
          alpha = fast_exp2(m_ref - mt);
          rescale = true;
        }
        m_ref = mt;
      }
      // P (and the output, if it is rescaled below) is free once PV(i-1) has
      // finished; PV(i) cannot start before p_full at the end of this tile
      if (i >= 1 && !(ok = warp_wait(smem_u32(&sm.p_empty), (i - 1) & 1, abort_flag, err))) break;
      tc_fence_after();
      {
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
        const bool live = m_ref > -INFINITY;
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float p0 = live ? fast_exp2(s[2 * c] - m_ref) : 0.f;
          const float p1 = live ? fast_exp2(s[2 * c + 1] - m_ref) : 0.f;
          ps[c & 3] += p0 + p1;
          const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
          pk[c] = *reinterpret_cast<const uint32_t*>(&pb);
        }
        tmem_st16(tmem + lane_base + kColP + 16 * g, pk);
        l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      }
      // a new reference maximum: rescale this warp's half of the output
      if (rescale) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          const uint32_t col = tmem + lane_base + kColO + 128 * g + 32 * c;
          tmem_ld32(col, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(col, o);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.p_full));
    }
    // ------------------------------------------------------- epilogue
    // The row sum is the sum over both key halves; each warp of a pair then
    // writes its 128 of this CTA's 256 output dims.
    if (ok && ntiles > 0 &&
        warp_wait(smem_u32(&sm.p_empty), (ntiles - 1) & 1, abort_flag, err)) {
      sm.pair_max[ntiles & 1][g][h] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.pair));
      if (warp_wait(smem_u32(&sm.pair), ntiles & 1, abort_flag, err)) {
        const float lt = l + sm.pair_max[ntiles & 1][g ^ 1][h];
        tc_fence_after();
        const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
        const bool head_ok = h < A.H;
        __nv_bfloat16* orow = A.out + (static_cast<long long>(r) * A.H + h) * 512 + dim0 + 128 * g;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(tmem + lane_base + kColO + 128 * g + 32 * c, o);
          if (head_ok) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const __nv_bfloat162 v =
                  __floats2bfloat162_rn(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
              pk[e] = *reinterpret_cast<const uint32_t*>(&v);
            }
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
        if (rank == 0 && g == 0 && head_ok && A.lse)
          A.lse[static_cast<long long>(r) * A.H + h] =
              lt > 0.f ? (m_ref + log2f(lt)) * 0.69314718055994531f : -INFINITY;
      }
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
  a.kv = static_cast<const __nv_bfloat16*>(kv);
  CUtensorMap tq, tqr;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cudaError_t e =
      make_tmap_2d(&tq, q, bf, 576, q_rows, 576 * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e == cudaSuccess)
    e = make_tmap_2d(&tqr, q, bf, 576, q_rows, 576 * 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(MlaSmem) + 1024;
  e = cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(2 * a.T);      // x has no 65535 limit; cluster pairs are consecutive x
  sparse_mla_kernel<<<grid, kMlaThreads, smem, st>>>(tq, tqr, a);
  return cudaGetLastError();
}

}  // namespace dsa

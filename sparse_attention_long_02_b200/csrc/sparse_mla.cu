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
// dims [256c, 256c+256). The logits are split by keys instead: of every tile
// of 64 selected slots, CTA c owns slots [32c, 32c+32) and forms their whole
// 576-dim logits itself (fp32 tensor-core sums, nothing exchanged below
// fp32), so each CTA holds all of Q (448 dims in TMEM, 128 in shared memory).
// Per tile:
//   1. six gather warps copy, with coalesced cp.async (through the block
//      table for the paged cache), the whole rows of the CTA's own 32 slots
//      and the CTA's 256 value dims of the peer's 32 slots, up to three tiles
//      ahead;
//   2. warp 1 issues S = Q K_own^T (M=128 heads, N=32 keys, K=576) into TMEM
//      as soon as the tile is gathered and the previous logits are read,
//      independently of the PV products;
//   3. eight softmax warps (thread = head, two warps per TMEM lane quarter,
//      16 keys each) take the tile maximum of their own keys; the two CTAs
//      swap their maxima one tile ahead (remote stores), so both use the same
//      running reference maximum, re-based only when it grows by more than 8
//      (log2 units, and only then is the output rescaled); P = exp2(s - m) is
//      written as bf16 into shared memory;
//   4. the exchange warp sends the CTA's half of P (8 KB) to the peer with one
//      bulk copy (the TMA engine), so both CTAs hold P for all 64 slots;
//   5. warp 1 issues O_c += P_own V_own + P_peer V_peer (M=128, N=256 dims,
//      K=32 + 32 keys), P and V both from shared memory (V in the MN-major
//      view of the gathered rows).
// The final output is O / l in bf16, l the sum over both CTAs' keys, and
// lse = (m + log2 l) * ln 2.
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kMlaThreads = 512;
constexpr int kTileKeys = 64;                   // selected slots per tile (both CTAs)
constexpr int kOwnKeys = 32;                    // slots per tile whose logits a CTA forms
constexpr int kStages = 3;
constexpr int kAtom = kOwnKeys * 128;           // 32 rows x 64 dims bf16, 128-B swizzled
constexpr int kOwnAtoms = 9;                    // 8 latent + 1 rope atom of the own rows
constexpr int kPeerAtoms = 4;                   // this CTA's 256 value dims of the peer's rows
constexpr int kQAtom = 128 * 128;               // 128 heads x 64 dims bf16
constexpr int kQTmemAtoms = 7;                  // Q dims [0, 448) live in TMEM
constexpr int kPHalf = 128 * kOwnKeys * 2;      // one CTA's P: 128 heads x 32 keys bf16
constexpr int kGatherWarps = 6;                 // warps 0, 2, 3, 12, 13, 14
constexpr int kSoftmaxWarps = 8;                // warps 4-11
constexpr int kExchangeWarp = 15;
constexpr uint32_t kColO = 0;                   // TMEM columns [0,256): output
constexpr uint32_t kColQ = 256;                 // [256,480): Q dims [0,448), bf16 pairs
constexpr uint32_t kColS = 480;                 // [480,512): logits of the own 32 keys
constexpr float kRebase = 8.0f;                 // lazy rescale threshold (log2 units)

struct MlaSmem {
  // stage = own rows (atoms 0-8), then the peer's rows' value dims (9-12)
  uint8_t kv[kStages][kOwnAtoms + kPeerAtoms][kAtom];
  uint8_t p[2][2][kPHalf];                      // [tile parity][slot half = owning CTA], 64-B swizzle
  uint8_t q_s[2][kQAtom];                       // Q dims [448,512) and [512,576)
  float mx[2][128];                             // the peer's tile maxima, by tile parity
  float pair_max[2][2][128];                    // [parity][key half][head]
  float l_peer[128];                            // the peer's row sums (end)
  unsigned valid[kStages];                      // selected bits of the own 32 slots
  unsigned long long q_full;                    // Q has landed in its staging slots
  unsigned long long q_ready;                   // Q is in TMEM (staging slots free)
  unsigned long long kv_full[kStages];
  unsigned long long kv_empty[kStages];
  unsigned long long s_full;
  unsigned long long s_empty;
  unsigned long long pair;                      // both key halves posted (max, or l at the end)
  unsigned long long mx_full[2];                // the peer's tile maximum has landed
  unsigned long long p_own[2];                  // this CTA's P half of a tile is written
  unsigned long long p_peer[2];                 // the peer's P half has landed
  unsigned long long p_acked[2];                // the peer holds the P half sent from here
  unsigned long long p_remote_free[2];          // the peer's PV no longer reads its p buffer
  unsigned long long pv_done[2];                // this CTA's PV of a tile has finished
  unsigned long long l_full;                    // the peer's row sums have landed
  unsigned long long o_done;
  uint32_t tmem_base;
  int abort_flag;
};

// Q's TMEM-bound atoms are staged in kv stages 1-2 and the P buffers, which
// are first written after Q has moved into TMEM.
constexpr size_t kQStageOff = sizeof(uint8_t[kOwnAtoms + kPeerAtoms][kAtom]);
static_assert(offsetof(MlaSmem, p) == kStages * kQStageOff, "P follows the ring");
static_assert(kQStageOff + kQTmemAtoms * kQAtom <=
                  offsetof(MlaSmem, q_s), "Q staging fits stages 1-2 and P");
static_assert(kQStageOff % 1024 == 0 && kAtom % 1024 == 0 && kPHalf % 1024 == 0,
              "1024-B aligned tiles");
static_assert(offsetof(MlaSmem, q_s) % 1024 == 0, "1024-B aligned Q atoms");
static_assert(sizeof(MlaSmem) + 1024 <= 232448, "fits the 227 KB of shared memory a CTA may use");

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
sparse_mla_kernel(const __grid_constant__ CUtensorMap tm_q, const MlaArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  MlaSmem& sm = *reinterpret_cast<MlaSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned* err = A.err;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const int c = static_cast<int>(rank);
  // query row (one cluster per row); dense prefill rows run longest first
  const int r = (A.dense && !A.block_table) ? A.T - 1 - static_cast<int>(blockIdx.x >> 1)
                                            : static_cast<int>(blockIdx.x >> 1);
  const int seq = A.block_table ? r / A.nq : 0;
  // keys a slot may name: the causal prefix of the query (paged) or the cache
  int limit = A.S;
  if (A.block_table) limit = A.seq_len[seq] - A.nq + (r % A.nq) + 1;
  // keys the row sees, and its slots: every such key in dense mode, else
  // the index set (only its first min(k, keys) entries when the sets hold
  // their selected slots first, the rest being -1; at least one, so that a
  // row that sees no key still writes its zero output and -inf lse)
  const int row_keys = A.block_table ? limit : min(A.q_pos0 + r + 1, A.S);
  const int nslots = A.dense ? row_keys : A.compact ? max(1, min(A.k, row_keys)) : A.k;
  const int ntiles = (nslots + kTileKeys - 1) / kTileKeys;
  const int* sel = A.dense ? nullptr : A.idx + static_cast<long long>(r) * A.k;
  const int warp = warp_id(), lane = lane_id();
  const int dim0 = 256 * c;                      // first value dim of this CTA
  // Both CTAs of the pair normally take the same early exit; if they did not,
  // the working one times out on the peer's barriers and still returns.
  const bool aborted = launch_aborted(err);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_ready), 4);         // the four warps that move Q into TMEM
    for (int i = 0; i < kStages; ++i) {
      // one cp.async-completion arrival per gathering thread + the slot writer
      mbar_init(smem_u32(&sm.kv_full[i]), 32 * kGatherWarps + 1);
      mbar_init(smem_u32(&sm.kv_empty[i]), 1);
    }
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.s_empty), kSoftmaxWarps);
    mbar_init(smem_u32(&sm.pair), kSoftmaxWarps);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.mx_full[b]), 128);        // one remote arrival per head
      mbar_init(smem_u32(&sm.p_own[b]), kSoftmaxWarps);
      mbar_init(smem_u32(&sm.p_peer[b]), 1);           // own expect_tx + the copied bytes
      mbar_init(smem_u32(&sm.p_acked[b]), 1);          // one arrival from the peer per use
      mbar_init(smem_u32(&sm.p_remote_free[b]), 1);    // one arrival from the peer per use
      mbar_init(smem_u32(&sm.pv_done[b]), 1);
    }
    mbar_init(smem_u32(&sm.l_full), 128);
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
  uint8_t* q_stage = reinterpret_cast<uint8_t*>(sm.kv[1]);

  const bool gather = warp == 0 || warp == 2 || warp == 3 || (warp >= 12 && warp <= 14);
  if (gather && !aborted) {
    // ------------------------------------------------------- gather warps
    // Whole rows of the own slots (72 x 16 B, latent atoms 0-7 and the rope
    // atom 8) and this CTA's 256 value dims of the peer's slots (32 x 16 B,
    // atoms 9-12), each 16-B chunk at its 128-B-swizzled place in its atom.
    const int gw = warp == 0 ? 0 : warp <= 3 ? warp - 1 : warp - 9;   // 0..5
    if (warp == 0 && lane == 0) {
      const uint32_t qf = smem_u32(&sm.q_full);
      mbar_expect_tx(qf, (kQTmemAtoms + 2) * kQAtom);
      for (int a = 0; a < kQTmemAtoms; ++a)
        tma_load_2d(smem_u32(q_stage + a * kQAtom), &tm_q, qf, 64 * a, r * A.H);
      for (int a = 0; a < 2; ++a)
        tma_load_2d(smem_u32(sm.q_s[a]), &tm_q, qf, 64 * (kQTmemAtoms + a), r * A.H);
    }
    // Two-deep prefetch: the slots of tile i+2 and the block-table entries
    // of tile i+1 are loading while tile i is issued. Lane l holds own slot
    // l and peer slot l of a tile.
    auto slot = [&](int j) { return j >= nslots ? -1 : A.dense ? j : __ldg(sel + j); };
    const int own0 = kOwnKeys * c + lane, peer0 = kOwnKeys * (c ^ 1) + lane;
    int vo = slot(own0), vp = slot(peer0);                                  // tile 0
    int bo = kv_block(A, vo, seq, limit), bp = kv_block(A, vp, seq, limit);
    int no = slot(kTileKeys + own0), np = slot(kTileKeys + peer0);          // tile 1
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % kStages;
      const int co = vo, cp = vp, po = bo, pp = bp;
      if (i + 1 < ntiles) {
        vo = no;
        vp = np;
        bo = kv_block(A, vo, seq, limit);
        bp = kv_block(A, vp, seq, limit);
      }
      if (i + 2 < ntiles) {
        no = slot((i + 2) * kTileKeys + own0);
        np = slot((i + 2) * kTileKeys + peer0);
      }
      const int ro = kv_row(A, co, po, limit), rp = kv_row(A, cp, pp, limit);
      // stages 1 and 2 hold Q's staging until it has moved into TMEM
      if (i == 1 && !warp_wait(smem_u32(&sm.q_ready), 0, abort_flag, err)) break;
      if (i >= kStages &&
          !warp_wait(smem_u32(&sm.kv_empty[st]), ((i / kStages) + 1) & 1, abort_flag, err))
        break;
      const uint32_t full = smem_u32(&sm.kv_full[st]);
      if (gw == 0) {
        const unsigned bits = __ballot_sync(0xffffffffu, ro >= 0);
        if (lane == 0) {
          sm.valid[st] = bits;
          mbar_arrive(full);
        }
      }
      const uint32_t base = smem_u32(sm.kv[st][0]);
      for (int row = gw; row < kOwnKeys; row += kGatherWarps) {
        const int pr = __shfl_sync(0xffffffffu, ro, row);
        const __nv_bfloat16* src = A.kv + static_cast<long long>(pr < 0 ? 0 : pr) * 576;
        const uint32_t nb = pr < 0 ? 0u : 16u;               // skipped slot: zero fill
#pragma unroll
        for (int k3 = 0; k3 < 3; ++k3) {
          const int ch = lane + 32 * k3;                    // 16-B chunk of the row, 0..71
          if (ch < 72)
            cp_async16(base + (ch >> 3) * kAtom + row * 128 + (((ch & 7) ^ (row & 7)) << 4),
                       src + ch * 8, nb);
        }
      }
      for (int row = gw; row < kOwnKeys; row += kGatherWarps) {
        const int pr = __shfl_sync(0xffffffffu, rp, row);
        const __nv_bfloat16* src = A.kv + static_cast<long long>(pr < 0 ? 0 : pr) * 576 + dim0;
        const uint32_t nb = pr < 0 ? 0u : 16u;
        cp_async16(base + (kOwnAtoms + (lane >> 3)) * kAtom + row * 128 +
                       (((lane & 7) ^ (row & 7)) << 4),
                   src + lane * 8, nb);
      }
      cp_async_arrive(full);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (warp == 0 && lane == 0) mbar_drain(smem_u32(&sm.q_full), 0);
  } else if (warp == kExchangeWarp && !aborted) {
    // ---------------------------------------------------- exchange warp
    // Tile i's P half goes from p[i&1][c] to the peer's p[i&1][c] in one bulk
    // copy once it is written and the peer's PV of tile i-2 no longer reads
    // that buffer. This warp also tells the peer when its half of tile i has
    // landed here (its source may be rewritten) and when this CTA's PV of a
    // tile has finished (it may send the tile two ahead). Cluster-scope
    // releases for P come from this warp only.
    if (lane == 0) {
      int sent = 0;
      bool ok = true;
      for (int j = 0; j < 2 && j < ntiles; ++j) mbar_expect_tx(smem_u32(&sm.p_peer[j]), kPHalf);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int b = i & 1;
        if (!(ok = mbar_wait(smem_u32(&sm.p_own[b]), (i >> 1) & 1, abort_flag, err))) break;
        if (i >= 2 &&
            !(ok = mbar_wait<true>(smem_u32(&sm.p_remote_free[b]), ((i - 2) >> 1) & 1, abort_flag,
                                   err)))
          break;
        bulk_copy_to_peer(mapa(smem_u32(sm.p[b][c]), peer), smem_u32(sm.p[b][c]), kPHalf,
                          mapa(smem_u32(&sm.p_peer[b]), peer));
        sent = i + 1;
        if (!(ok = mbar_wait<true>(smem_u32(&sm.p_peer[b]), (i >> 1) & 1, abort_flag, err))) break;
        mbar_arrive_remote(mapa(smem_u32(&sm.p_acked[b]), peer));
        if (i + 2 < ntiles) mbar_expect_tx(smem_u32(&sm.p_peer[b]), kPHalf);     // tile i+2
        if (i >= 1) {
          const int j = i - 1;
          if (!(ok = mbar_wait(smem_u32(&sm.pv_done[j & 1]), (j >> 1) & 1, abort_flag, err))) break;
          mbar_arrive_remote(mapa(smem_u32(&sm.p_remote_free[j & 1]), peer));
        }
      }
      // A copy reads this CTA's P buffer until it lands: wait for the peer's
      // word on the last two before this CTA may leave (the softmax warps
      // waited for every earlier one before rewriting a buffer).
      for (int j = sent > 2 ? sent - 2 : 0; j < sent; ++j) {
        const uint32_t bar = smem_u32(&sm.p_acked[j & 1]);
        if (!mbar_wait<true>(bar, (j >> 1) & 1, abort_flag, err)) mbar_drain(bar, (j >> 1) & 1);
      }
    }
  } else if (warp == 1 && !aborted) {
    // ------------------------------------------------------- MMA thread
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(128, kOwnKeys, false);
      const uint32_t id_pv = idesc_bf16(128, 256, true);
      bool ok = mbar_wait(smem_u32(&sm.q_ready), 0, abort_flag, err);
      // debug: o_done completes only after the commit below, so this bounded
      // wait runs out and both CTAs leave through their give-up paths
      if (ok && (debug_bits(err) & kDbgStallMla))
        ok = mbar_wait(smem_u32(&sm.o_done), 0, abort_flag, err);
      auto issue_qk = [&](int i) {
        const int st = i % kStages;
        fence_proxy_async_smem();         // cp.async (generic) writes -> tensor-core reads
        tc_fence_after();
        const uint32_t d = tmem + kColS;
        for (int a = 0; a < kOwnAtoms; ++a) {
          const uint64_t kd = sdesc_sw128(smem_u32(sm.kv[st][a]), 0, 1024);
          if (a < kQTmemAtoms) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)        // 4 x K=16 dims (8 TMEM columns of Q)
              mma_bf16_ts(d, tmem + kColQ + 32 * a + 8 * kk, kd + 2 * kk, id_qk,
                          (a > 0 || kk > 0) ? 1u : 0u);
          } else {
            const uint64_t qd = sdesc_sw128(smem_u32(sm.q_s[a - kQTmemAtoms]), 0, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(d, qd + 2 * kk, kd + 2 * kk, id_qk, 1u);
          }
        }
        mma_commit(smem_u32(&sm.s_full));
      };
      auto issue_pv = [&](int i) {
        const int st = i % kStages, b = i & 1;
        tc_fence_after();
        // keys of CTA h's slots: P from p[b][h], V from this CTA's own rows
        // (h == c: their atoms 4c..4c+3) or from the peer rows' value dims
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t vbase =
              smem_u32(sm.kv[st][h == c ? 4 * c : kOwnAtoms]);
          const uint64_t vdesc = sdesc_sw128(vbase, kAtom, 1024);
          const uint64_t pdesc = sdesc_sw64(smem_u32(sm.p[b][h]), 512);
#pragma unroll
          for (int kk = 0; kk < kOwnKeys / 16; ++kk)          // 16 keys: 32 B of P, 2 KB of V
            mma_bf16(tmem + kColO, pdesc + 2 * kk, vdesc + (kk * 2048 >> 4), id_pv,
                     (i > 0 || h > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(smem_u32(&sm.pv_done[b]));
        mma_commit(smem_u32(&sm.kv_empty[st]));
      };
      // QK(i) needs its gathered tile and the softmax warps' read of tile
      // i-1's logits; PV(i) needs both P halves of tile i. Neither waits for
      // the other: this thread polls both and issues whichever is ready, so a
      // late P half from the peer holds back only the PV, never the next
      // tile's logits. Both run in tile order; a stall of either longer than
      // the wait limit gives up like any bounded wait.
      int nq = 0, np = 0;
      unsigned long long t_last = globaltimer();
      while (ok && np < ntiles) {
        bool moved = false;
        if (nq < ntiles && mbar_test_wait(smem_u32(&sm.kv_full[nq % kStages]), (nq / kStages) & 1) &&
            (nq == 0 || mbar_test_wait(smem_u32(&sm.s_empty), (nq - 1) & 1))) {
          issue_qk(nq++);
          moved = true;
        }
        if (np < nq && mbar_test_wait(smem_u32(&sm.p_own[np & 1]), (np >> 1) & 1) &&
            mbar_test_wait_cluster(smem_u32(&sm.p_peer[np & 1]), (np >> 1) & 1)) {
          issue_pv(np++);
          moved = true;
        }
        if (moved) {
          t_last = globaltimer();
        } else if (*abort_flag) {
          ok = false;
        } else if (globaltimer() - t_last > kWaitLimitNs) {
          *abort_flag = 1;
          raise_error(err, kErrTimeout);
          ok = false;
        }
      }
      mma_commit(smem_u32(&sm.o_done));
      mbar_drain(smem_u32(&sm.o_done), 0);
    }
  } else if (warp >= 4 && warp < 4 + kSoftmaxWarps && !aborted) {
    // ------------------------------------------------- softmax warps
    const int g = (warp - 4) >> 2;                      // key half of the own slots
    const int h = 32 * (warp & 3) + lane;               // head = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    if (g == 0) {
      // Move this head's row of Q dims [0, 448) from its staging atoms into
      // TMEM (bf16 pairs, lane = head).
      if ((ok = warp_wait(smem_u32(&sm.q_full), 0, abort_flag, err))) {
#pragma unroll 1
        for (int a = 0; a < kQTmemAtoms; ++a) {
          const uint4* row = reinterpret_cast<const uint4*>(q_stage + a * kQAtom + h * 128);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t pk[16];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint4 v = row[(4 * half + cc) ^ (h & 7)];
              pk[4 * cc] = v.x;
              pk[4 * cc + 1] = v.y;
              pk[4 * cc + 2] = v.z;
              pk[4 * cc + 3] = v.w;
            }
            tmem_st16(tmem + lane_base + kColQ + 32 * a + 16 * half, pk);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.q_ready));
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    // Tile j's logits of this warp's 16 keys (log2 units, unselected slots
    // -inf) and the CTA's maximum over its 32 keys, which goes to the peer.
    float s[16];
    float mo = -INFINITY;                               // this CTA's maximum of the tile
    auto load_tile = [&](int j) -> bool {
      const int st = j % kStages;
      if (!warp_wait(smem_u32(&sm.kv_full[st]), (j / kStages) & 1, abort_flag, err)) return false;
      if (!warp_wait(smem_u32(&sm.s_full), j & 1, abort_flag, err)) return false;
      tc_fence_after();
      tmem_ld16(tmem + lane_base + kColS + 16 * g, s);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.s_empty));
      // which of the own slots are selected (written by the gather warps
      // before kv_full(j))
      const unsigned valid = sm.valid[st] >> (16 * g);
      float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        s[e] = ((valid >> e) & 1u) ? s[e] * A.sm_scale_log2 : -INFINITY;
        pm[e & 3] = fmaxf(pm[e & 3], s[e]);
      }
      sm.pair_max[j & 1][g][h] = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.pair));
      if (!warp_wait(smem_u32(&sm.pair), j & 1, abort_flag, err)) return false;
      mo = fmaxf(sm.pair_max[j & 1][0][h], sm.pair_max[j & 1][1][h]);
      if (g == 0) {                                     // one store per head
        st_cluster_f32(mapa(smem_u32(&sm.mx[j & 1][h]), peer), mo);
        mbar_arrive_remote(mapa(smem_u32(&sm.mx_full[j & 1]), peer));
      }
      return true;
    };
    if (ok && ntiles > 0) ok = load_tile(0);
    for (int i = 0; ok && i < ntiles; ++i) {
      const int b = i & 1;
      // the peer's maximum of tile i, sent while it finished tile i-1
      if (!(ok = warp_wait<true>(smem_u32(&sm.mx_full[b]), (i >> 1) & 1, abort_flag, err))) break;
      const float mt = fmaxf(mo, sm.mx[b][h]);
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_ref + kRebase) {        // also the first tile with a selected key
        if (m_ref > -INFINITY) {
          alpha = fast_exp2(m_ref - mt);
          rescale = true;
        }
        m_ref = mt;
      }
      // p[b] is free once this CTA's PV of tile i-2 has read it and the peer
      // holds the half sent from it
      if (i >= 2 &&
          !(ok = warp_wait(smem_u32(&sm.pv_done[b]), ((i - 2) >> 1) & 1, abort_flag, err) &&
                 warp_wait<true>(smem_u32(&sm.p_acked[b]), ((i - 2) >> 1) & 1, abort_flag, err)))
        break;
      {
        const bool live = m_ref > -INFINITY;
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float p0 = live ? fast_exp2(s[2 * e] - m_ref) : 0.f;
          const float p1 = live ? fast_exp2(s[2 * e + 1] - m_ref) : 0.f;
          ps[e & 3] += p0 + p1;
          const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
          pk[e] = *reinterpret_cast<const uint32_t*>(&pb);
        }
        // row h of this CTA's P half: 64 B, 16-B chunk q (keys 8q..8q+7) at
        // chunk q ^ ((h / 2) % 4)
        uint4* prow = reinterpret_cast<uint4*>(sm.p[b][c] + h * 64);
        prow[(2 * g) ^ ((h >> 1) & 3)] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        prow[(2 * g + 1) ^ ((h >> 1) & 3)] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      }
      // a new reference maximum: once PV of tile i-1 has finished, rescale
      // this warp's half of the output. The TMEM loads and stores are
      // warp-collective, so the whole warp takes the branch when any head
      // re-bases (the others scale by alpha = 1).
      if (__any_sync(0xffffffffu, rescale)) {
        if (i >= 1 && !(ok = warp_wait(smem_u32(&sm.pv_done[(i - 1) & 1]), ((i - 1) >> 1) & 1,
                                       abort_flag, err)))
          break;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float o[32];
          const uint32_t col = tmem + lane_base + kColO + 128 * g + 32 * cc;
          tmem_ld32(col, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(col, o);
        }
      }
      fence_proxy_async_smem();           // P (generic writes) -> MMA and bulk-copy reads
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.p_own[b]));
      // the next tile's maximum goes out while the peer finishes this one
      if (i + 1 < ntiles && !(ok = load_tile(i + 1))) break;
    }
    // ------------------------------------------------------- epilogue
    // l over both key halves of this CTA, then over both CTAs; each warp of a
    // pair writes its 128 of this CTA's 256 output dims.
    const int last = ntiles - 1;
    if (ok && ntiles > 0 &&
        warp_wait(smem_u32(&sm.pv_done[last & 1]), (last >> 1) & 1, abort_flag, err)) {
      sm.pair_max[ntiles & 1][g][h] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.pair));
      if (warp_wait(smem_u32(&sm.pair), ntiles & 1, abort_flag, err)) {
        const float lc = sm.pair_max[ntiles & 1][0][h] + sm.pair_max[ntiles & 1][1][h];
        if (g == 0) {
          st_cluster_f32(mapa(smem_u32(&sm.l_peer[h]), peer), lc);
          mbar_arrive_remote(mapa(smem_u32(&sm.l_full), peer));
        }
        if (warp_wait<true>(smem_u32(&sm.l_full), 0, abort_flag, err)) {
          const float lt = lc + sm.l_peer[h];
          tc_fence_after();
          const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
          const bool head_ok = h < A.H;
          __nv_bfloat16* orow =
              A.out + (static_cast<long long>(r) * A.H + h) * 512 + dim0 + 128 * g;
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            float o[32];
            tmem_ld32(tmem + lane_base + kColO + 128 * g + 32 * cc, o);
            if (head_ok) {
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const __nv_bfloat162 v =
                    __floats2bfloat162_rn(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
                pk[e] = *reinterpret_cast<const uint32_t*>(&v);
              }
              uint4* dst = reinterpret_cast<uint4*>(orow + 32 * cc);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            }
          }
          if (c == 0 && g == 0 && head_ok && A.lse)
            A.lse[static_cast<long long>(r) * A.H + h] =
                lt > 0.f ? (m_ref + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        }
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
  CUtensorMap tq;
  cudaError_t e = make_tmap_2d(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 576, q_rows, 576 * 2, 64,
                               128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(MlaSmem) + 1024;
  e = cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(2 * a.T);      // x has no 65535 limit; cluster pairs are consecutive x
  sparse_mla_kernel<<<grid, kMlaThreads, smem, st>>>(tq, a);
  return cudaGetLastError();
}

}  // namespace dsa

// indexer.cu -- lightning indexer scores on sm_100a tensor cores.
//
// Computes, for every causal (query t, key s) pair,
//     I[t,s] = k_scale[s] * sum_h (w[t,h] * scale * q_scale[t]) * ReLU(x[t,h,s]),
//     x[t,h,s] = sum_{d<128} q8[t,h,d] * k8[s,d]           (e4m3 x e4m3 -> f32)
// which equals sum_h w[t,h] * ReLU(scale * qf[t,h] . kf[s]) because the
// scales are positive. Method: "DeepSeek-V3.2-Exp 模型优势与 DSA 工作原理",
// section 4, step 2 (dot product, mask, scale, per-head weight); FP8 and
// ReLU: "m.gxzdkb.com/media/457.html", section "秘密武器".
//
// Tiling: keys sit on the MMA's M dimension (128 keys = 128 TMEM lanes),
// queries x heads on N (QB queries x HI heads <= 256 columns), K = 128 is
// four e4m3 MMAs of K = 32. Two TMEM accumulator buffers and two epilogue
// groups let the MMA of key tile i+1 run under the epilogue of tile i.
//
// Epilogue, HI >= 32 (the DSA configs): a thread reads its lane quarter's
// accumulator with 16-lane TMEM loads, which give it four key rows x every
// fourth column, so the folded weights w * scale * q_scale of its columns
// (64 values for 256 columns) stay in registers for the whole CTA and each
// serves four keys. ReLU and the weighted sum over its heads run in packed
// f32x2 FMAs; a two-step butterfly over the four lanes that share the rows
// completes each row's head sum. (Reading the weights from shared memory per
// element instead kept the shared-memory pipe ~70% busy and cost ~27% of the
// kernel.) HI < 32: a thread owns one key row and reduces whole queries in
// registers.
//
// Warp roles (320 threads = 10 warps): warp 0 = TMA producer, warp 1 = MMA
// issuer and TMEM owner, warps 2-9 = epilogue, group (w-2)/4 = TMEM buffer.
// A warp may only touch TMEM lanes 32*(w%4) .. +31, and each run of four
// consecutive warps covers the four lane quarters.
#include "common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kIdxThreads = 320;
static_assert(kIdxThreads / 32 == 2 + 8, "producer, MMA issuer and 8 epilogue warps");

// Order-preserving 32-bit key of a float score (larger score, larger key).
__device__ __forceinline__ uint32_t score_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
// The float threshold equivalent to an order-key threshold: score_key(x) >= k
// exactly when x >= key_threshold(k), for every score the epilogue forms (no
// NaN, and no -0: its sums start at +0, and x - x rounds to +0). Keys at or
// below that of -inf keep every score; keys above that of +inf keep none
// (the result is a NaN, which compares false).
__device__ __forceinline__ float key_threshold(uint32_t k) {
  if (k <= 0x007fffffu) return -INFINITY;
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
constexpr int kKeyTile = 128;      // keys per MMA tile (M)
constexpr int kStages = 4;         // key-tile ring depth
constexpr int kKTileBytes = kKeyTile * 128;

// Filter mode: each CTA first appends its candidates to lists in shared memory
// (this many bytes in all) and copies them out once at the end. For HI >= 32
// each epilogue warp keeps its own list per query, with its counts in
// registers, so an append needs no atomic; otherwise the lists are per query.
constexpr int kCandSmemBytes = 64 * 1024;

struct IdxSmem {
  // operand tiles first (1024-B aligned by construction of the offsets)
  uint8_t q[256 * 128];                 // B operand: QB*HI rows x 128 B
  uint8_t k[kStages][kKTileBytes];      // A operand ring
  float w[256];                         // w[t,h]*scale*q_scale[t] for the CTA's queries
  // the same for HI >= 32, by 32-column block b and lane group t0 = lane % 4:
  // wt[b][t0][k] = w[32b + 4k + t0] (rows padded to 12 so that the four
  // groups' 16-B loads fall in distinct banks)
  float wt[8][4][12];
  float tau[64];                        // filter mode: the CTA's queries' thresholds
  uint32_t cand_n[64];                  // filter mode: entries in each query's list
  unsigned long long q_full;
  unsigned long long k_full[kStages];
  unsigned long long k_empty[kStages];
  unsigned long long t_full[2];
  unsigned long long t_empty[2];
  unsigned long long mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

// Prefill: one CTA per SM, so the epilogue may keep its 64 weights in
// registers (about 164 a thread). Paged: two CTAs per SM, which caps a thread
// at 102 registers (96 used; the weights past the second block are read from
// shared memory).
template <int HI, bool PAGED>
__global__ void __launch_bounds__(kIdxThreads, PAGED ? 2 : 1)
indexer_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const IndexerArgs a) {
  constexpr int QB = (256 / HI) < 64 ? (256 / HI) : 64;   // queries per CTA (prefill)
  constexpr int kCapS = kCandSmemBytes / (QB * 8);         // shared-memory entries per query
  constexpr int kCapW = kCandSmemBytes / (8 * QB * 8);     // per epilogue warp and query (HI >= 32)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  IdxSmem& sm = *reinterpret_cast<IdxSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // filter mode: [QB][kCapS] order keys, then [QB][kCapS] key positions
  uint32_t* cs_key = reinterpret_cast<uint32_t*>(&sm + 1);
  int* cs_idx = reinterpret_cast<int*>(cs_key + QB * kCapS);
  unsigned* err = a.err;
  if (launch_aborted(err)) return;

  // ------------------------------------------------------------ work unit
  // Queries [q0, q0+nqb) of sequence `seq` (decode) or of the prefill block;
  // key tiles [tile0, tile1) of that sequence.
  int q0, nqb, seq = 0;
  long long pos0;            // position of query q0
  long long key_limit;       // keys of this sequence / cache
  if (PAGED) {
    seq = blockIdx.x;
    const int len = a.seq_len[seq];
    nqb = a.nq;
    q0 = seq * a.nq;
    pos0 = static_cast<long long>(len) - a.nq;
    key_limit = len;
  } else {
    const int qb = gridDim.x - 1 - blockIdx.x;     // longest rows first
    q0 = qb * QB;
    nqb = min(QB, a.T - q0);
    pos0 = static_cast<long long>(a.q_pos0) + q0;
    key_limit = a.S;
  }
  const long long last_key = min(pos0 + nqb - 1, key_limit - 1);
  const int ntiles_total = static_cast<int>((last_key + kKeyTile) / kKeyTile);
  const int tile0 = blockIdx.y * a.tiles_per_cta;
  const int tile1 = min(ntiles_total, tile0 + a.tiles_per_cta);
  if (nqb <= 0 || last_key < 0 || tile0 >= tile1) return;
  const int ntiles = tile1 - tile0;
  const int ncol = a.n_mma;                 // MMA N = padded QB*HI (or nq*HI)
  const uint32_t idesc = idesc_e4m3(128, ncol);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.q_full), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&sm.k_full[i]), 1);
      mbar_init(smem_u32(&sm.k_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.t_full[i]), 1);
      mbar_init(smem_u32(&sm.t_empty[i]), 4);
    }
    mbar_init(smem_u32(&sm.mma_done), 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (!PAGED && a.tau && threadIdx.x < QB) {
    const int qq = threadIdx.x;
    sm.cand_n[qq] = 0;
    sm.tau[qq] = key_threshold(qq < nqb ? a.tau[q0 + qq] : 0xffffffffu);
  }
  // folded per-(query, head) weights: w * scale * q_scale
  for (int j = threadIdx.x; j < ncol; j += blockDim.x) {
    const int qq = j / HI, h = j % HI;
    float v = 0.f;
    if (qq < nqb) {
      const long long t = q0 + qq;
      const float qs = a.q_scale ? a.q_scale[t] : 1.f;
      v = a.w[t * HI + h] * (a.scale * qs);
    }
    sm.w[j] = v;
    sm.wt[j >> 5][j & 3][(j & 31) >> 2] = v;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), a.tmem_cols);
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
      mbar_expect_tx(smem_u32(&sm.q_full), a.q_box_rows * 128);
      tma_load_2d(smem_u32(sm.q), &tm_q, smem_u32(&sm.q_full), 0, q0 * HI);
      int issued = 0;
      // paged: the two physical blocks of a key tile, loaded a tile ahead so
      // that the block-table read is off the copy-issue path
      auto blocks = [&](int i, int (&pb)[2]) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int lb = 2 * (tile0 + i) + half;          // logical block
          pb[half] = (i < ntiles && lb * 64 < key_limit)
                         ? __ldg(a.block_table + static_cast<long long>(seq) * a.max_blocks + lb)
                         : 0;
        }
      };
      int pb_next[2] = {0, 0};
      if (PAGED) blocks(0, pb_next);
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % kStages;
        int pb[2] = {pb_next[0], pb_next[1]};
        if (PAGED) blocks(i + 1, pb_next);
        if (i >= kStages &&
            !mbar_wait(smem_u32(&sm.k_empty[st]), ((i / kStages) + 1) & 1, abort_flag, err))
          break;
        const uint32_t full = smem_u32(&sm.k_full[st]);
        mbar_expect_tx(full, kKTileBytes);
        const int tile = tile0 + i;
        if (PAGED) {
          for (int half = 0; half < 2; ++half) {
            if (pb[half] < 0 || pb[half] >= a.nblk) {
              raise_error(err, kErrBounds);
              pb[half] = 0;
            }
            tma_load_2d(smem_u32(sm.k[st]) + half * 64 * 128, &tm_k, full, 0, pb[half] * 64);
          }
        } else {
          tma_load_2d(smem_u32(sm.k[st]), &tm_k, full, 0, tile * kKeyTile);
        }
        ++issued;
      }
      // make sure no copy is still landing when the CTA leaves
      for (int i = max(0, issued - kStages); i < issued; ++i)
        mbar_drain(smem_u32(&sm.k_full[i % kStages]), (i / kStages) & 1);
      mbar_drain(smem_u32(&sm.q_full), 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(smem_u32(&sm.q_full), 0, abort_flag, err);
      // debug: mma_done completes only after the commit below, so this
      // bounded wait runs out and the CTA leaves through its give-up path
      if (ok && (debug_bits(err) & kDbgStallIndexer))
        ok = mbar_wait(smem_u32(&sm.mma_done), 0, abort_flag, err);
      const uint64_t bdesc = sdesc_sw128(smem_u32(sm.q), 0, 1024);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int st = i % kStages, buf = i & 1;
        if (!mbar_wait(smem_u32(&sm.k_full[st]), (i / kStages) & 1, abort_flag, err)) break;
        if (i >= 2 && !mbar_wait(smem_u32(&sm.t_empty[buf]), ((i >> 1) + 1) & 1, abort_flag, err))
          break;
        tc_fence_after();
        const uint64_t adesc = sdesc_sw128(smem_u32(sm.k[st]), 0, 1024);
        const uint32_t d = tmem + buf * ncol;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)     // 4 x K=32 (32 bytes each)
          mma_f8f6f4(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0);
        mma_commit(smem_u32(&sm.k_empty[st]));
        mma_commit(smem_u32(&sm.t_full[buf]));
      }
      mma_commit(smem_u32(&sm.mma_done));
      mbar_drain(smem_u32(&sm.mma_done), 0);
    }
  } else if (warp >= 2) {
    // --------------------------------------------------------- epilogue
    const int g = (warp - 2) >> 2;                 // epilogue group = TMEM buffer
    // accumulator row (key in tile) whose score this thread emits: its own
    // TMEM lane, or for HI >= 32 the lane the head-sum butterfly below leaves
    // with it
    const int t0 = lane & 3, t1 = lane >> 2;
    const int row = 32 * (warp & 3) + (HI >= 32 ? t1 + 8 * (t0 & 1) + 16 * (t0 >> 1) : lane);
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    // k_scale of this thread's key in tile i, fetched one tile ahead so the
    // load's latency hides behind the previous tile's epilogue
    auto key_scale = [&](int i) -> float {
      const long long s = static_cast<long long>(tile0 + i) * kKeyTile + row;
      if (!a.k_scale || i >= ntiles || s >= key_limit) return 1.f;
      if (PAGED) {
        int pb = a.block_table[static_cast<long long>(seq) * a.max_blocks + (s >> 6)];
        pb = (pb < 0 || pb >= a.nblk) ? 0 : pb;
        return __ldg(a.k_scale + static_cast<long long>(pb) * 64 + (s & 63));
      }
      return __ldg(a.k_scale + s);
    };
    float ks_next = key_scale(g);
    // HI >= 32: the folded weights of this thread's columns, 32c + 4k + t0
    // (c < 8, k < 8), in registers for the whole CTA
    // paged (decode) rows keep the first two blocks' weights in registers and
    // read the rest from shared memory, so that two CTAs fit on an SM
    constexpr int kWB = PAGED ? 2 : 8;
    float wreg[8 * kWB];
    if constexpr (HI >= 32) {
#pragma unroll
      for (int b = 0; b < 8; ++b)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (b < kWB) wreg[8 * b + k] = b < ncol / 32 ? sm.wt[b][t0][k] : 0.f;
    }
    const unsigned lane_lt = (1u << lane) - 1u;
    // filter mode, HI >= 32: the queries' thresholds in registers
    float tau_r[HI >= 32 ? QB : 1];
#pragma unroll
    for (int e = 0; e < (HI >= 32 ? QB : 1); ++e) tau_r[e] = sm.tau[e];
    const int ew = warp - 2;                       // epilogue warp 0..7
    unsigned wcnt[HI >= 32 ? QB : 1];              // this warp's appends per query (HI >= 32)
#pragma unroll
    for (int e = 0; e < (HI >= 32 ? QB : 1); ++e) wcnt[e] = 0;
    for (int i = g; i < ntiles; i += 2) {
      const float ks = ks_next;
      ks_next = key_scale(i + 2);
      if (!warp_wait(smem_u32(&sm.t_full[g]), (i >> 1) & 1, abort_flag, err)) break;
      tc_fence_after();
      const long long s = static_cast<long long>(tile0 + i) * kKeyTile + row;   // logical key
      const bool key_ok = s < key_limit;
      // filter mode: the key is causal for query qq when qq >= sd
      const int sd = static_cast<int>(s - pos0);
      const uint32_t taddr = tmem + lane_base + g * ncol;
      // hand the buffer back to the MMA as soon as its last columns are in
      // registers, so the next MMA into it overlaps the tail of this epilogue
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.t_empty[g]));
      };
      // Called by the whole warp with the same qq. Scores mode writes the
      // row; filter mode appends (order key, key) of every score at or above
      // the query's threshold to a list in shared memory (this warp's own for
      // HI >= 32, else the query's, one shared atomic per warp and query),
      // or, once that list is full, straight to the row's list in global
      // memory.
      auto emit = [&](int qq, float acc) {
        if (qq >= nqb) return;
        const long long t = q0 + qq;
        const long long pos = pos0 + qq;
        if (!PAGED && a.tau) {
          const float sc = acc * ks;
          const bool keep = key_ok && sd <= qq && sc >= (HI >= 32 ? tau_r[qq] : sm.tau[qq]);
          const unsigned ball = __ballot_sync(0xffffffffu, keep);
          const uint32_t key = score_key(sc);
          if constexpr (HI >= 32) {
            if (ball) {
              const unsigned base = wcnt[qq];
              const unsigned slot = base + __popc(ball & lane_lt);
              const bool local = slot < static_cast<unsigned>(kCapW);
              uint32_t* lk = cs_key + (ew * QB + qq) * kCapW;
              int* li = cs_idx + (ew * QB + qq) * kCapW;
              if (keep && local) {
                lk[slot] = key;
                li[slot] = static_cast<int>(s);
              }
              wcnt[qq] = base + __popc(ball);
              const unsigned over = base + __popc(ball) > static_cast<unsigned>(kCapW)
                                        ? __ballot_sync(0xffffffffu, keep && !local)
                                        : 0u;
              if (over) {
                unsigned gb = 0;
                if (lane == 0) gb = atomicAdd(a.cand_count + t, static_cast<unsigned>(__popc(over)));
                gb = __shfl_sync(0xffffffffu, gb, 0) + __popc(over & lane_lt);
                if (keep && !local && gb < static_cast<unsigned>(a.cand_cap)) {
                  a.cand_key[t * a.cand_cap + gb] = key;
                  a.cand_idx[t * a.cand_cap + gb] = static_cast<int>(s);
                }
              }
            }
            return;
          }
          if (ball) {
            unsigned base = 0;
            if (lane == 0) base = atomicAdd(&sm.cand_n[qq], static_cast<unsigned>(__popc(ball)));
            base = __shfl_sync(0xffffffffu, base, 0);
            const unsigned slot = base + __popc(ball & lane_lt);
            const bool local = slot < static_cast<unsigned>(kCapS);
            if (keep && local) {
              cs_key[qq * kCapS + slot] = key;
              cs_idx[qq * kCapS + slot] = static_cast<int>(s);
            }
            // the warp's appends overflow the shared list only when its last
            // slot does (warp-uniform test)
            const unsigned over = base + __popc(ball) > static_cast<unsigned>(kCapS)
                                      ? __ballot_sync(0xffffffffu, keep && !local)
                                      : 0u;
            if (over) {
              unsigned gb = 0;
              if (lane == 0) gb = atomicAdd(a.cand_count + t, static_cast<unsigned>(__popc(over)));
              gb = __shfl_sync(0xffffffffu, gb, 0) + __popc(over & lane_lt);
              if (keep && !local && gb < static_cast<unsigned>(a.cand_cap)) {
                a.cand_key[t * a.cand_cap + gb] = key;
                a.cand_idx[t * a.cand_cap + gb] = static_cast<int>(s);
              }
            }
          }
          return;
        }
        if (!key_ok) return;
        float* out = a.scores + t * a.ld;
        out[s] = (s <= pos) ? acc * ks : -INFINITY;
      };
      if constexpr (HI >= 32) {
        // 32 columns per pair of 16-lane TMEM loads: this thread holds
        // columns 4k + t0 (k < 8) of the rows t1, t1+8, 16+t1, 24+t1 of its
        // lane quarter, so each weight in wreg serves four keys. ReLU, then
        // the weighted sum over its 8 heads of each row (packed f32x2 FMAs);
        // at the end of a query a butterfly over the four lanes t0 = 0..3
        // sums the four lane groups' heads and leaves lane t0 with the total
        // of row t1 + 8 (t0 % 2) + 16 (t0 / 2).
        const uint32_t ta = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + g * ncol;
        const uint32_t tb = ta + (16u << 16);
        float2 acc[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (c >= ncol / 32) break;
          float v[32];
          tmem_ld_16x128b_x8_pair(ta + c * 32, tb + c * 32, v);
          if (c == ncol / 32 - 1) release();
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const float4 w4 =
                c < kWB ? make_float4(wreg[(8 * c + 4 * m) % (8 * kWB)], wreg[(8 * c + 4 * m + 1) % (8 * kWB)],
                                      wreg[(8 * c + 4 * m + 2) % (8 * kWB)], wreg[(8 * c + 4 * m + 3) % (8 * kWB)])
                        : reinterpret_cast<const float4*>(sm.wt[c][t0])[m];
            const float2 wa = make_float2(w4.x, w4.y), wb = make_float2(w4.z, w4.w);
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {         // row rr: v[16 (rr/2) + 2k + rr%2]
              const float* x = v + 16 * (rr >> 1) + (rr & 1);
              const int k = 4 * m;
              acc[rr] = __ffma2_rn(wa, make_float2(fmaxf(x[2 * k], 0.f), fmaxf(x[2 * k + 2], 0.f)),
                                   acc[rr]);
              acc[rr] = __ffma2_rn(wb, make_float2(fmaxf(x[2 * k + 4], 0.f), fmaxf(x[2 * k + 6], 0.f)),
                                   acc[rr]);
            }
          }
          if ((c * 32 + 32) % HI == 0) {
            float p[4];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
              p[rr] = acc[rr].x + acc[rr].y;
              acc[rr] = make_float2(0.f, 0.f);
            }
            // lanes t0 and t0^1 swap the rows the other keeps: even t0 keeps
            // rows {0, 2} (t1, 16+t1), odd t0 rows {1, 3}
            const bool odd = t0 & 1;
            const float k0 = odd ? p[1] : p[0], k1 = odd ? p[3] : p[2];
            const float s0 = odd ? p[0] : p[1], s1 = odd ? p[2] : p[3];
            const float q0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 1);
            const float q1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 1);
            // then t0 and t0^2: t0 < 2 keeps the first, t0 >= 2 the second
            const bool hi2 = t0 >> 1;
            const float tot = (hi2 ? q1 : q0) + __shfl_xor_sync(0xffffffffu, hi2 ? q0 : q1, 2);
            emit((c * 32) / HI, tot);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < ncol / 32; ++c) {
          float v[32];
          tmem_ld32(taddr + c * 32, v);
          if (c == ncol / 32 - 1) release();
          const float* wp = sm.w + c * 32;
#pragma unroll
          for (int qq = 0; qq < 32 / HI; ++qq) {
            float acc = 0.f;
#pragma unroll
            for (int h = 0; h < HI; ++h)
              acc = fmaf(wp[qq * HI + h], fmaxf(v[qq * HI + h], 0.f), acc);
            emit(c * (32 / HI) + qq, acc);
          }
        }
      }
    }
    // filter mode, HI >= 32: this warp's lists go to the rows' lists in
    // global memory, one atomic per query
    if constexpr (HI >= 32) {
      if (!PAGED && a.tau) {
        __syncwarp();
#pragma unroll
        for (int qq = 0; qq < QB; ++qq) {
          const unsigned n = min(wcnt[qq], static_cast<unsigned>(kCapW));
          if (qq >= nqb || n == 0) continue;
          const long long t = q0 + qq;
          unsigned gb = 0;
          if (lane == 0) gb = atomicAdd(a.cand_count + t, n);
          gb = __shfl_sync(0xffffffffu, gb, 0);
          const uint32_t* lk = cs_key + (ew * QB + qq) * kCapW;
          const int* li = cs_idx + (ew * QB + qq) * kCapW;
          for (unsigned j = lane; j < n; j += 32) {
            if (gb + j < static_cast<unsigned>(a.cand_cap)) {
              a.cand_key[t * a.cand_cap + gb + j] = lk[j];
              a.cand_idx[t * a.cand_cap + gb + j] = li[j];
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.tmem_cols);
  }
  // filter mode, HI < 32: each query's shared-memory list goes to the row's
  // list in global memory with one atomic (entries past the row's capacity
  // are dropped; the count still tells the select kernel the row overflowed)
  if (HI < 32 && !PAGED && a.tau) {
    for (int qq = warp; qq < nqb; qq += kIdxThreads / 32) {
      const unsigned n = min(sm.cand_n[qq], static_cast<unsigned>(kCapS));
      if (n == 0) continue;
      const long long t = q0 + qq;
      unsigned gb = 0;
      if (lane == 0) gb = atomicAdd(a.cand_count + t, n);
      gb = __shfl_sync(0xffffffffu, gb, 0);
      for (unsigned j = lane; j < n; j += 32) {
        if (gb + j < static_cast<unsigned>(a.cand_cap)) {
          a.cand_key[t * a.cand_cap + gb + j] = cs_key[qq * kCapS + j];
          a.cand_idx[t * a.cand_cap + gb + j] = cs_idx[qq * kCapS + j];
        }
      }
    }
  }
}

template <int HI, bool PAGED>
cudaError_t launch_one(const CUtensorMap& tq, const CUtensorMap& tk, const IndexerArgs& a,
                       dim3 grid, cudaStream_t st) {
  // Prefill: above half the SM's shared memory, so one CTA per SM (a second
  // would only queue on the TMEM allocation). Paged (decode): two CTAs per SM
  // (96 registers, at most 256 TMEM columns each), so a batch's key slices
  // fill the SMs in one wave instead of 1.7.
  const size_t smem = (PAGED ? sizeof(IdxSmem) + 1024
                             : std::max<size_t>(sizeof(IdxSmem) + 1024, 120 * 1024)) +
                      (a.tau ? kCandSmemBytes : 0);
  auto kern = indexer_kernel<HI, PAGED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  // the whole shared carveout, so shared memory never keeps a CTA off an SM
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  kern<<<grid, kIdxThreads, smem, st>>>(tq, tk, a);
  return cudaGetLastError();
}

template <bool PAGED>
cudaError_t launch_hi(int Hi, const CUtensorMap& tq, const CUtensorMap& tk, const IndexerArgs& a,
                      dim3 grid, cudaStream_t st) {
  switch (Hi) {
    case 1: return launch_one<1, PAGED>(tq, tk, a, grid, st);
    case 2: return launch_one<2, PAGED>(tq, tk, a, grid, st);
    case 4: return launch_one<4, PAGED>(tq, tk, a, grid, st);
    case 8: return launch_one<8, PAGED>(tq, tk, a, grid, st);
    case 16: return launch_one<16, PAGED>(tq, tk, a, grid, st);
    case 32: return launch_one<32, PAGED>(tq, tk, a, grid, st);
    case 64: return launch_one<64, PAGED>(tq, tk, a, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int indexer_queries_per_cta(int Hi) {
  const int qb = 256 / Hi;
  return qb < 64 ? qb : 64;
}

// Key tiles per CTA: prefill rows are long, so units of 128 tiles (16384 keys)
// amortise each CTA's setup; decode keeps 64 so that B = 64 sequences still
// spread over every SM.
static int indexer_tiles_per_cta(bool paged) { return paged ? 64 : 128; }

cudaError_t launch_indexer(const IndexerArgs& a_in, const void* q8, const void* k8,
                           long long k_rows, cudaStream_t st) {
  IndexerArgs a = a_in;
  const bool paged = a.block_table != nullptr;
  const int qb = paged ? a.nq : indexer_queries_per_cta(a.Hi);
  int n = qb * a.Hi;
  n = (n + 63) / 64 * 64;                   // the epilogue reads TMEM 64 columns at a time
  if (n < 64 || n > 256) return cudaErrorInvalidValue;
  a.n_mma = n;
  a.q_box_rows = n;
  a.tmem_cols = 2 * n <= 32 ? 32 : 2 * n <= 64 ? 64 : 2 * n <= 128 ? 128 : 2 * n <= 256 ? 256 : 512;
  a.tiles_per_cta = indexer_tiles_per_cta(paged);

  CUtensorMap tq, tk;
  const long long q_rows = paged ? static_cast<long long>(a.B) * a.nq * a.Hi
                                 : static_cast<long long>(a.T) * a.Hi;
  cudaError_t e = make_tmap_2d(&tq, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, q_rows, 128, 128, n,
                               CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&tk, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, k_rows, 128, 128,
                   paged ? 64 : kKeyTile, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;

  dim3 grid;
  if (paged) {
    const int max_tiles = (a.max_ctx + kKeyTile - 1) / kKeyTile;
    grid = dim3(a.B, (max_tiles + a.tiles_per_cta - 1) / a.tiles_per_cta);
    return launch_hi<true>(a.Hi, tq, tk, a, grid, st);
  }
  const int nblocks = (a.T + qb - 1) / qb;
  const long long max_key = std::min<long long>(static_cast<long long>(a.q_pos0) + a.T, a.S);
  const int max_tiles = static_cast<int>((max_key + kKeyTile - 1) / kKeyTile);
  grid = dim3(nblocks, (max_tiles + a.tiles_per_cta - 1) / a.tiles_per_cta);
  return launch_hi<false>(a.Hi, tq, tk, a, grid, st);
}

}  // namespace dsa

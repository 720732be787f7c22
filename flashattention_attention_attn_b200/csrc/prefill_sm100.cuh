// prefill_sm100.cuh - fused causal / non-causal GQA attention forward for
// sm_100a: TMA tile loads, tcgen05 MMAs with accumulators in tensor memory,
// online softmax in registers, warp-specialised roles.
//
// What it computes is the blockwise scheme of the page "Snelle
// attention-kernels en operatorfusie versnellen AI-modellen" (the-ai.news),
// section "FlashAttention-type aandacht en gepagineerde aandacht": for each
// key/value block, form that block's scores, update the running softmax
// statistics (row max, row sum) and accumulate the output on chip; the full
// score matrix is never written out.
//
// CTA = two 128-row query tiles (rows m0..m0+255) of one (batch, q-head).
//   warps 0-3  softmax for query tile 0 (thread r owns row r = TMEM lane r)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer (Q once, then a K ring and a V ring)
//   warp  9    MMA issuer (one thread): S_t = Q_t K^T, O_t += P_t V
//   warps 10-11 idle; with them the CTA is three whole warpgroups, so that
//   warpgroup 2 can hand registers to the softmax warpgroups (setmaxnreg)
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   S_0 cols [0,128), S_1 [128,256): fp32 scores; after the softmax the same
//   columns hold P as packed bf16 (64 columns), the A operand of P V.
//   O_0 [256, 256+D), O_1 [256+D, 256+2D): fp32 output accumulators.
// The two query tiles ping-pong: while the softmax warps of one tile work,
// the tensor core runs the other tile's MMAs.  The tile with more key tiles
// (the lead) has its copies and, in every key iteration, its MMAs issued
// first: its chain S -> softmax -> P V -> next S is the CTA's critical path.
// K / V tiles are loaded with an L2 evict_last policy (the other heads of the
// GQA group and the later query blocks read them again), Q and O with
// evict_first.
// The kernel is launched as a programmatic dependent of the previous grid on
// the stream: barrier set-up, the tensor-memory allocation and (dense mode) L2
// prefetches of the first tiles happen before the grid-dependency wait.  The
// epilogue stages each warp's 32 output rows in the tile's (by then free) Q
// buffer and stores them coalesced.
//
// Softmax statistics are kept in the log2 domain (s * scale * log2 e) and the
// exponentials use ex2.  The row max used as reference is only moved (and O
// rescaled by exp2(m_old - m_new)) when the new max exceeds it by more than
// kRescaleThreshold; otherwise P carries values up to 2^threshold, which fp32
// accumulation and bf16 P (same exponent range as fp32) absorb.  O and the row
// sum always share the same reference, so the final O / l is unchanged.
#pragma once

#include "sm100_ptx.cuh"

namespace attn {
namespace prefill {

constexpr int kBM = 128;               // rows per query tile (= TMEM lanes)
constexpr int kBN = 128;               // keys per K/V tile
constexpr int kThreads = 384;          // 12 warps: three warpgroups
// Registers per thread after the split (setmaxnreg): the softmax warpgroups
// hold a 128-score row per thread, warpgroup 2 (producer, MMA issuer, two
// idle warps) needs few.  The kernel is compiled for 168 per thread at
// launch (65536 / 384, in steps of 8); the split must not add up to more,
// or the increase would wait forever -- the host checks the compiled count
// before the first launch (kLaunchRegs).
constexpr int kSoftmaxRegs = 216;
constexpr int kOtherRegs = 72;
constexpr int kLaunchRegs = 168;
static_assert(2 * kSoftmaxRegs + kOtherRegs <= 3 * kLaunchRegs, "register split exceeds the launch allocation");
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Config {
  static constexpr int kChunks = D / 64;                     // 128-byte swizzle chunks per row
  static constexpr int kStages = (D == 64) ? 4 : 2;          // K ring depth = V ring depth
  static constexpr uint32_t kTileBytes = kBM * D * 2;        // one Q / K / V tile (bf16)
  static constexpr uint32_t kChunkBytes = kBM * 128;         // 128 rows x 128 bytes
};

template <int D>
struct __align__(1024) Smem {
  using C = Config<D>;
  __nv_bfloat16 q[2][C::kChunks][kBM * 64];
  __nv_bfloat16 k[C::kStages][C::kChunks][kBN * 64];
  __nv_bfloat16 v[C::kStages][C::kChunks][kBN * 64];
  uint64_t q_full[2];
  uint64_t k_full[C::kStages], v_full[C::kStages];
  // kv_done[i % kStages] completes when key iteration i has finished with
  // K(i) and V(i - 1): one commit per iteration frees a K slot and a V slot
  uint64_t kv_done[C::kStages];
  uint64_t s_full[2], p_full[2], o_full[2];
  uint64_t mma_done;
  uint64_t v_tail;  // paged: V tile holding the sequence end, before its tail is cleared
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t smem_bytes() {
  return sizeof(Smem<D>) + 1024;  // + slack to align the dynamic base to 1024
}

// How queries and keys are laid out.
constexpr int kDense = 0;   // [B, T, H, D] / [B, S, H, D]
constexpr int kVarlen = 1;  // packed [total, H, D], offsets from cu_q / cu_k
constexpr int kPaged = 2;   // packed queries; keys and values in a paged pool

struct Params {
  float* lse;             // [B, Hq, T] (dense) / [Hq, total_q] (packed), or nullptr
  __nv_bfloat16* o;       // output base (row stores of ragged packed tiles)
  const int32_t* cu_q;    // packed: [B + 1] prefix sums of query lengths
  const int32_t* cu_k;    // varlen: [B + 1] prefix sums of key lengths
  const int32_t* block_table;  // paged: [B, max_blocks] physical 16-token blocks
  const int32_t* seq_lens;     // paged: [B] cached tokens (keys) per sequence
  int max_blocks;
  int num_blocks;              // paged: pool size; block ids outside [0, num_blocks) are masked
  int B, Hq, Hkv, T, S;   // dense: T, S; varlen: T = max query length
  int total_q;            // varlen: rows of the packed query tensor
  int causal;
  float scale_log2;  // scale * log2(e)
  int num_mblocks;   // ceil(T / 256)
  int items;         // packed, B <= 32: grid = Hq x items (see below); 0: grid = Hq x B x num_mblocks
};

// Keys visible to the query tile with rows [r0, r0 + 128) (ragged T clipped)
// as a number of kBN-wide K/V tiles; 0 when no row of it sees any key.
__device__ __forceinline__ int kv_tiles_for(int r0, int T, int S, int causal) {
  if (r0 >= T) return 0;
  const int r1 = min(r0 + kBM, T);
  int kmax = S - 1;
  if (causal) kmax = min(kmax, r1 - 1 + (S - T));
  if (kmax < 0) return 0;
  return kmax / kBN + 1;
}

// MODE kVarlen / kPaged: packed sequences (no padding).  The query / output
// maps then cover [total, H, D] as batch 1 and each CTA takes its sequence's
// row offset and length from cu_q.  kVarlen takes key rows from cu_k the
// same way; kPaged reads every 128-key tile as eight 16-token blocks through
// the block table (pool maps of [tokens, Hkv * D], box 64 x 16).  In kPaged
// mode a sequence length is clamped to the table row's capacity and a block
// id outside [0, num_blocks) is not loaded and its 16 keys are masked; both
// set a bit of the device status word.
template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_fwd_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const Params p) {
  using C = Config<D>;
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work tile: heaviest (last) query blocks first; adjacent CTAs are adjacent
  // q heads of one (block, batch) so the heads sharing a KV head run together.
  const int per_mb = p.Hq * p.B;
  int mb = p.num_mblocks - 1 - static_cast<int>(blockIdx.x) / per_mb;
  const int rem = static_cast<int>(blockIdx.x) % per_mb;
  const int h = rem % p.Hq;
  int b = rem / p.Hq;
  const int hk = h / (p.Hq / p.Hkv);
  int m0 = mb * 2 * kBM;
  constexpr bool VARLEN = MODE != kDense;  // packed queries and outputs

  // Setup that reads no global memory (barriers, tensor memory, descriptor
  // prefetch) overlaps the tail of the previous grid on the stream; this
  // kernel is launched as its programmatic dependent.
  if (warp == kWarpLoad && lane == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.q_full[t], 1);
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.p_full[t], 4);  // one arrive per softmax warp
      mbar_init(&sm.o_full[t], 1);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.kv_done[s], 1);
      mbar_init(&sm.v_full[s], 1);
    }
    mbar_init(&sm.mma_done, 1);
    mbar_init(&sm.v_tail, 1);
    sm.abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if constexpr (MODE == kDense) {
      // The first tiles into L2 while the previous grid finishes (the
      // shapes are known without reading memory in this mode).
      if (kv_tiles_for(m0, p.T, p.S, p.causal) + kv_tiles_for(m0 + kBM, p.T, p.S, p.causal) > 0) {
        for (int t = 0; t < 2; ++t)
          if (m0 + t * kBM < p.T)
            for (int c = 0; c < C::kChunks; ++c) tma_prefetch_l2_4d(&tmQ, c * 64, h, m0 + t * kBM, b);
        for (int c = 0; c < C::kChunks; ++c) {
          tma_prefetch_l2_4d(&tmK, c * 64, hk, 0, b);
          tma_prefetch_l2_4d(&tmV, c * 64, hk, 0, b);
        }
      }
    }
  }
  if (!VARLEN && warp == 0) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  grid_dependency_wait();
  grid_launch_dependents();

  int T = p.T, S = p.S, qoff = 0, koff = 0, bc = b;  // bc: batch coordinate of the maps
  if constexpr (VARLEN) {
    if (p.items > 0) {
      // Compact grid: CTA -> work item blockIdx / Hq -> (sequence, query
      // block), without the blocks past a sequence's end.  Packed prefill:
      // the order of the full grid (top query blocks first, sequences
      // ascending), so the heaviest blocks start first.  Lane i holds
      // sequence i's block count; every warp finds the same item.
      const int len = (lane < p.B) ? p.cu_q[lane + 1] - p.cu_q[lane] : 0;
      const int nblocks = (len + 2 * kBM - 1) / (2 * kBM);
      int left = static_cast<int>(blockIdx.x) / p.Hq;
      b = -1;
      if constexpr (MODE == kPaged) {
        // Chunked prefill: sequence-major (a sequence's query blocks, top
        // first, are adjacent), so that its blocks read the same keys and
        // values from L2 while they are there.
        int incl = nblocks;  // inclusive prefix sum of the block counts
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int excl = incl - nblocks;
        const uint32_t m = __ballot_sync(0xffffffffu, left >= excl && left < incl);
        if (m != 0) {
          b = __ffs(m) - 1;
          mb = __shfl_sync(0xffffffffu, nblocks, b) - 1 - (left - __shfl_sync(0xffffffffu, excl, b));
        }
      } else {
        for (int k = p.num_mblocks - 1; k >= 0 && b < 0; --k) {
          uint32_t m = __ballot_sync(0xffffffffu, nblocks > k);
          const int c = __popc(m);
          if (left < c) {
            for (int i = 0; i < left; ++i) m &= m - 1;  // drop the first `left` set bits
            b = __ffs(m) - 1;
            mb = k;
          } else {
            left -= c;
          }
        }
      }
      if (b < 0) return;  // past the last item (the grid is an upper bound)
      m0 = mb * 2 * kBM;
    }
    qoff = p.cu_q[b];
    T = p.cu_q[b + 1] - qoff;
    if constexpr (MODE == kPaged) {
      // clamped to what the table row can name (flagged when outside)
      S = p.seq_lens[b];
      if (S < 0 || S > p.max_blocks * 16) {
        if (threadIdx.x == 0 && h == 0) atomicOr(&g_devstatus, kDevStatusBadSeqLen);
        S = S < 0 ? 0 : p.max_blocks * 16;
      }
    } else {
      koff = p.cu_k[b];
      S = p.cu_k[b + 1] - koff;
    }
    bc = 0;
    // A query block past the sequence (uniform over the CTA) leaves before
    // it allocates tensor memory: packed batches of short sequences have many.
    if (m0 >= T) return;
    if (warp == 0) {
      tmem_alloc(&sm.tmem_base, kTmemCols);
      tmem_relinquish();
    }
  }
  const int n0 = kv_tiles_for(m0, T, S, p.causal);
  const int n1 = kv_tiles_for(m0 + kBM, T, S, p.causal);
  const int n_max = max(n0, n1);
  // The lead tile is the one with more key tiles (tile 1 of a causal block
  // unless it lies past the end): its chain S -> softmax -> P V -> next S is
  // the CTA's critical path, so its copies and MMAs go first.
  const int lead = (n1 >= n0 && n1 > 0) ? 1 : 0;

  // The first copies leave before the CTA-wide barrier, in the order the
  // MMAs need them: Q of the lead tile, K tile 0, Q of the other tile, V
  // tile 0 (K / V only for contiguous keys: paged tiles need the warp's
  // table reads).
  const int pre = (MODE != kPaged && n_max > 0) ? 1 : 0;  // K / V tiles issued here
  if (warp == kWarpLoad && lane == 0) {
    const int nt[2] = {n0, n1};
    auto load_q = [&](int t) {
      if (nt[t] == 0) return;
      mbar_arrive_expect_tx(&sm.q_full[t], C::kTileBytes);
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d_hint(sm.q[t][c], &tmQ, &sm.q_full[t], c * 64, h, qoff + m0 + t * kBM, bc, l2_policy_evict_first());
    };
    load_q(lead);
    if constexpr (MODE != kPaged) {
      if (pre) {
        mbar_arrive_expect_tx(&sm.k_full[0], C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d_hint(sm.k[0][c], &tmK, &sm.k_full[0], c * 64, hk, koff, bc, l2_policy_evict_last());
      }
    }
    load_q(1 - lead);
    if constexpr (MODE != kPaged) {
      if (pre) {
        mbar_arrive_expect_tx(&sm.v_full[0], C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d_hint(sm.v[0][c], &tmV, &sm.v_full[0], c * 64, hk, koff, bc, l2_policy_evict_last());
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp >= 8) {
  // Warpgroup 2 (producer, MMA issuer, two idle warps) hands registers to
  // the two softmax warpgroups, which hold a 128-score row per thread.
  reg_dealloc<kOtherRegs>();
  if (warp == kWarpLoad) {
    // ------------------------------ producer ------------------------------
    // The whole warp runs the loop; lane 0 waits on the barriers.  Contiguous
    // tiles take one copy per 64-column chunk (lane 0).  Paged tiles take one
    // copy per 16-token block and chunk: lane L reads table entry L and issues
    // the copy of (chunk L / 8, block L % 8), so the 16 copies of a tile leave
    // in one warp instruction instead of one after another.
    const int nt[2] = {n0, n1};
    int k_issued = pre, v_issued = pre;  // K / V tiles whose loads were issued
    const uint64_t kv_pol = l2_policy_evict_last();  // K / V tiles are read again by the other heads and blocks
    bool tail_issued = false;
    constexpr int kBlocks = kBN / 16;     // 16-token blocks per tile
    const int cl = lane / kBlocks, il = lane % kBlocks;  // paged: this lane's (chunk, block)
    for (int j = pre; j < n_max; ++j) {
      const int s = j % C::kStages;
      const uint32_t ph = (j / C::kStages) & 1;
      int nblk = kBlocks;    // 16-token blocks of this tile inside the sequence
      int valid = kBN;       // keys of this tile inside the sequence
      int my_id = 0;         // paged: physical block of this lane's copy
      uint32_t bad = 0;      // paged: blocks of this tile whose id lies outside the pool
      if constexpr (MODE == kPaged) {
        valid = min(kBN, S - j * kBN);
        nblk = (valid + 15) / 16;
        const int mine = (lane < nblk) ? __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks +
                                               j * kBlocks + lane)
                                       : 0;
        bad = __ballot_sync(0xffffffffu, lane < nblk && static_cast<unsigned>(mine) >=
                                                            static_cast<unsigned>(p.num_blocks));
        my_id = __shfl_sync(0xffffffffu, mine, il);
        if (bad && lane == 0) atomicOr(&g_devstatus, kDevStatusBadBlock);
      }
      // blocks outside the pool are not loaded (the softmax masks their keys)
      const bool my_copy = MODE == kPaged && cl < C::kChunks && il < nblk && !((bad >> il) & 1u);
      const uint32_t tile_bytes = static_cast<uint32_t>(nblk - __popc(bad)) * 16 * D * 2;
      // Rows of blocks outside the pool in a free V slot are cleared, so that
      // a zero weight cannot meet a NaN left there.
      auto clear_bad_rows = [&]() {
        for (int i = lane; i < kBlocks * 16 * C::kChunks * 8; i += 32) {
          const int unit = i & 7, c = (i >> 3) % C::kChunks, r = (i >> 3) / C::kChunks;
          if ((bad >> (r / 16)) & 1u)
            *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(sm.v[s][c]) + r * 128 + unit * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
      };
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(&sm.kv_done[s], ph ^ 1, abort_flag);  // iteration j - kStages freed K's slot
        if (ok) {
          mbar_arrive_expect_tx(&sm.k_full[s], tile_bytes);
          if constexpr (MODE != kPaged) {
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_4d_hint(sm.k[s][c], &tmK, &sm.k_full[s], c * 64, hk, koff + j * kBN, bc, kv_pol);
          }
        }
      }
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
      if (my_copy)
        tma_load_2d_hint(reinterpret_cast<uint8_t*>(sm.k[s][cl]) + il * 16 * 128, &tmK, &sm.k_full[s],
                    hk * D + cl * 64, my_id * 16, kv_pol);
      if (lane == 0) {
        k_issued = j + 1;
        // V(j) reuses V(j - kStages)'s slot, freed by iteration j - kStages + 1
        if (j >= C::kStages) {
          const int it = j - C::kStages + 1;
          ok = mbar_wait(&sm.kv_done[it % C::kStages], (it / C::kStages) & 1, abort_flag);
        }
      }
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
      if (MODE == kPaged && valid < kBN) {
        // The tile holding the sequence end: its V copy completes on v_tail;
        // then the rows past the end (pool slots that may hold anything,
        // even NaN, and blocks not loaded) are cleared so that a zero weight
        // cannot meet a NaN, and only then is the tile handed to the MMA.
        if (lane == 0) mbar_arrive_expect_tx(&sm.v_tail, tile_bytes);
        __syncwarp();
        if (my_copy)
          tma_load_2d_hint(reinterpret_cast<uint8_t*>(sm.v[s][cl]) + il * 16 * 128, &tmV, &sm.v_tail,
                      hk * D + cl * 64, my_id * 16, kv_pol);
        tail_issued = true;
        ok = __shfl_sync(0xffffffffu, mbar_wait(&sm.v_tail, 0, abort_flag) ? 1 : 0, 0) != 0;
        if (!ok) break;
        for (int i = lane; i < (kBN - valid) * C::kChunks * 8; i += 32) {
          const int unit = i & 7, c = (i >> 3) % C::kChunks, r = valid + (i >> 3) / C::kChunks;
          *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(sm.v[s][c]) + r * 128 + unit * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        if (bad) clear_bad_rows();
        fence_proxy_async_smem();  // the generic writes before the tensor core reads the tile
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.v_full[s]);
      } else {
        if (MODE == kPaged && bad) {
          clear_bad_rows();
          fence_proxy_async_smem();  // before the arrive that hands the tile to the MMA
          __syncwarp();
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.v_full[s], tile_bytes);
          if constexpr (MODE != kPaged) {
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_4d_hint(sm.v[s][c], &tmV, &sm.v_full[s], c * 64, hk, koff + j * kBN, bc, kv_pol);
          }
        }
        __syncwarp();
        if (my_copy)
          tma_load_2d_hint(reinterpret_cast<uint8_t*>(sm.v[s][cl]) + il * 16 * 128, &tmV, &sm.v_full[s],
                      hk * D + cl * 64, my_id * 16, kv_pol);
      }
      v_issued = j + 1;
    }
    if (lane == 0 && *abort_flag) {
      // Let the copies already issued land before shared memory is released.
      for (int t = 0; t < 2; ++t)
        if (nt[t] > 0) mbar_wait_drain(&sm.q_full[t], 0);
      for (int j = max(0, k_issued - C::kStages); j < k_issued; ++j)
        mbar_wait_drain(&sm.k_full[j % C::kStages], (j / C::kStages) & 1);
      for (int j = max(0, v_issued - C::kStages); j < v_issued; ++j)
        mbar_wait_drain(&sm.v_full[j % C::kStages], (j / C::kStages) & 1);
      if (tail_issued) mbar_wait_drain(&sm.v_tail, 0);
    }
  } else if (warp == kWarpMma) {
    // ---------------------------- MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_bf16(kBM, kBN, 0, 0);  // Q, K both K-major
      constexpr uint32_t idesc_pv = make_idesc_bf16(kBM, D, 0, 1);    // P (TMEM), V MN-major
      const int nt[2] = {n0, n1};
      const int ord[2] = {lead, 1 - lead};
      bool ok = true;

      // O_t += P_t(jj) V(jj).  Every commit and every wait costs this thread
      // ~100 cycles on the critical path of a P hand-off, so V(jj) is waited
      // for once per iteration (wait_v: the tile that comes first) and O_t
      // is committed only after the tile's last P V (last).
      auto issue_pv = [&](int t, int jj, bool wait_v, bool last) -> bool {
        const int s = jj % C::kStages;
        if (wait_v && !mbar_wait(&sm.v_full[s], (jj / C::kStages) & 1, abort_flag)) return false;
        const uint32_t tS = tmem + t * kBN;
        const uint32_t tO = tmem + 2 * kBN + t * D;
        const uint32_t vbase = smem_u32(sm.v[s][0]);
        if (!mbar_wait(&sm.p_full[t], jj & 1, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // 16 keys per step: 16 rows x 128 B further into each V chunk;
          // LBO = distance between 64-wide d chunks, SBO = 8 rows x 128 B.
          const uint64_t bdesc = make_sdesc_sw128(vbase + kk * 16 * 128, C::kChunkBytes, 1024);
          umma_ts(tO, tS + kk * 8, bdesc, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        if (last) umma_commit(&sm.o_full[t]);
        return true;
      };

      for (int j = 0; j < n_max && ok; ++j) {
        const int s = j % C::kStages;
        if (!(ok = mbar_wait(&sm.k_full[s], (j / C::kStages) & 1, abort_flag))) break;
        tc_fence_after();
        for (int i = 0; i < 2 && ok; ++i) {
          const int t = ord[i];
          // the previous P_t must be consumed before S_t is overwritten
          if (j >= 1 && j - 1 < nt[t]) ok = issue_pv(t, j - 1, i == 0, j == nt[t]);
          if (ok && j == 0 && nt[t] > 0) ok = mbar_wait(&sm.q_full[t], 0, abort_flag);
          if (ok && j < nt[t]) {
            const uint32_t tS = tmem + t * kBN;
            const uint32_t qbase = smem_u32(sm.q[t][0]);
            const uint32_t kbase = smem_u32(sm.k[s][0]);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk / 4) * C::kChunkBytes + (kk % 4) * 32;
              const uint64_t adesc = make_sdesc_sw128(qbase + off, 16, 1024);
              const uint64_t bdesc = make_sdesc_sw128(kbase + off, 16, 1024);
              umma_ss(tS, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
            }
            umma_commit(&sm.s_full[t]);
          }
        }
        if (!ok) break;
        umma_commit(&sm.kv_done[s]);  // K(j) and V(j - 1) are free
      }
      if (ok && n_max > 0) {
        const int jl = n_max - 1;
        for (int i = 0; i < 2 && ok; ++i)
          if (jl < nt[ord[i]]) ok = issue_pv(ord[i], jl, i == 0, true);

      }
      // Every MMA issued above is complete once mma_done fires; after an
      // abort this keeps tensor memory allocated until they have finished.
      umma_commit(&sm.mma_done);
      mbar_wait_drain(&sm.mma_done, 0);
    }
  }
  } else {
    reg_alloc<kSoftmaxRegs>();
    // ------------------------------ softmax -------------------------------
    const int t = warp >> 2;              // query tile of this warpgroup
    const int r = threadIdx.x & 127;      // row within the tile = TMEM lane
    const int row = m0 + t * kBM + r;
    const int nt = t ? n1 : n0;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * kBN;
    const uint32_t tO = tmem + lane_off + 2 * kBN + t * D;
    const int visible = p.causal ? min(S, row + (S - T) + 1) : S;
    const float sl2 = p.scale_log2;

    float m_used = -INFINITY;  // reference max, log2 domain
    float l = 0.f;             // running row sum relative to m_used
    bool ok = true;
    // paged: lane i < 8 holds the table entry of block i of the next key
    // tile (loaded one tile ahead); blocks outside the pool are masked
    auto table_entry = [&](int jj) -> int {
      const int nb = min(kBN / 16, (S - jj * kBN + 15) / 16);
      return lane < nb ? __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks + jj * (kBN / 16) + lane)
                       : 0;
    };
    int entry_next = (MODE == kPaged && nt > 0) ? table_entry(0) : 0;
    for (int j = 0; j < nt; ++j) {
      const int entry = entry_next;
      if (MODE == kPaged && j + 1 < nt) entry_next = table_entry(j + 1);
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[t], j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float s[kBN];
      {
        uint32_t u[kBN];
        tmem_ld128_sync(tS, u);
#pragma unroll
        for (int i = 0; i < kBN; ++i) s[i] = __uint_as_float(u[i]);
      }
      const int lim = visible - j * kBN;  // visible columns of this tile
      if (lim < kBN) {
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          if (i >= lim) s[i] = -INFINITY;
      }
      if constexpr (MODE == kPaged) {
        const int nb = min(kBN / 16, (S - j * kBN + 15) / 16);
        const uint32_t bad = __ballot_sync(0xffffffffu, lane < nb && static_cast<unsigned>(entry) >=
                                                                         static_cast<unsigned>(p.num_blocks));
        if (bad) {  // warp-uniform
#pragma unroll
          for (int g = 0; g < kBN / 16; ++g)
            if ((bad >> g) & 1u) {
#pragma unroll
              for (int i = 0; i < 16; ++i) s[g * 16 + i] = -INFINITY;
            }
        }
      }
      // Row max with 3-input max: 8 independent chains of 16 scores each.
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        mx8[k] = fmaxf(s[k], s[k + 8]);
#pragma unroll
        for (int m = 1; m < kBN / 16; ++m) mx8[k] = fmax3(mx8[k], s[k + 16 * m], s[k + 16 * m + 8]);
      }
      const float mx = fmaxf(fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), mx8[6]), mx8[7]);
      const float m_new = fmaxf(m_used, mx * sl2);
      const bool move = m_new - m_used > kRescaleThreshold;  // false while both are -inf (NaN)
      if (__any_sync(0xffffffffu, move)) {
        // O_t already holds P V of earlier tiles (their MMAs completed before
        // this tile's S was committed) unless the row has seen no key yet.
        const bool rescale = move && m_used != -INFINITY;
        if (__any_sync(0xffffffffu, rescale)) {
          // tcgen05.ld / st are warp-wide: the whole warp takes the round
          // trip, rows that keep their reference with a factor of 1.
          const float alpha = rescale ? ex2_approx(m_used - m_new) : 1.f;
          l *= alpha;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tmem_ld32_sync(tO + c * 32, u);
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
            tmem_st_x32(tO + c * 32, u);
          }
        }
        if (move) m_used = m_new;
      }
      const float mref = (m_used == -INFINITY) ? 0.f : m_used;
      // x = s * scale * log2(e) - m and the row sum in packed fp32 pairs;
      // P = 2^x goes to tensor memory as bf16 pairs, chunk by chunk.
      const float2 c2 = make_float2(sl2, sl2);
      const float2 nm2 = make_float2(-mref, -mref);
      float2 sum4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 x = __ffma2_rn(make_float2(s[c * 32 + 2 * i], s[c * 32 + 2 * i + 1]), c2, nm2);
          const float2 pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          sum4[i & 3] = __fadd2_rn(sum4[i & 3], pp);
          pk[i] = pack_bf16x2(pp.x, pp.y);
        }
        tmem_st_x16(tS + c * 16, pk);  // P overwrites the first 64 columns of S
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[t]);
      const float2 s01 = __fadd2_rn(sum4[0], sum4[1]);
      const float2 s23 = __fadd2_rn(sum4[2], sum4[3]);
      const float2 sall = __fadd2_rn(s01, s23);
      l += sall.x + sall.y;
    }

    if (ok && nt > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_full[t], 0, abort_flag));  // one commit, after the last P V
      tc_fence_after();
    }
    // Epilogue: O / l -> bf16.  Each warp stages its 32 rows in this tile's
    // Q buffer (free: the tile's last QK^T completed before o_full fired),
    // 16-byte chunks XOR-swizzled by row so that neither the row-wise writes
    // nor the chunk-wise reads conflict on banks, then copies them out with
    // whole rows per group of lanes (coalesced), skipping rows past the end.
    // No wait on any copy: the CTA can retire at once.
    {
      constexpr int kRowBytes = D * 2;
      constexpr int kChunksPerRow = kRowBytes / 16;  // 16 (D = 128) or 8 (D = 64)
      constexpr int kRowsPerPass = 32 / kChunksPerRow;
      const float inv_l = (l > 0.f) ? 1.0f / l : 0.f;
      const bool have_o = ok && nt > 0;  // warp-uniform: tcgen05.ld is warp-wide
      uint8_t* stage = reinterpret_cast<uint8_t*>(sm.q[t][0]) + (warp & 3) * 32 * kRowBytes;
      uint8_t* my_row = stage + lane * kRowBytes;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        if (have_o) {
          tmem_ld32_sync(tO + c * 32, u);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(u[2 * i]) * inv_l, __uint_as_float(u[2 * i + 1]) * inv_l);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = (c * 4 + q4) ^ (lane & (kChunksPerRow - 1));
          *reinterpret_cast<uint4*>(my_row + chunk * 16) =
              make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
      }
      __syncwarp();
      const int warp_row0 = t * kBM + (warp & 3) * 32;  // first row of this warp within the CTA's block
      const int chunk = lane % kChunksPerRow;
      const uint64_t o_pol = l2_policy_evict_first();  // O is written once
#pragma unroll 4
      for (int pass = 0; pass < 32 / kRowsPerPass; ++pass) {
        const int rl = pass * kRowsPerPass + lane / kChunksPerRow;  // row within the warp's 32
        const int rrow = m0 + warp_row0 + rl;                       // row within the sequence
        const uint4 val =
            *reinterpret_cast<const uint4*>(stage + rl * kRowBytes + ((chunk ^ (rl & (kChunksPerRow - 1))) * 16));
        if (rrow < T) {
          const size_t orow = VARLEN ? static_cast<size_t>(qoff) + rrow : static_cast<size_t>(b) * T + rrow;
          st_global_v4_hint(reinterpret_cast<uint4*>(p.o + (orow * p.Hq + h) * D) + chunk, val, o_pol);
        }
      }
    }
    if (p.lse != nullptr && row < T) {
      const float lse = (l > 0.f) ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const size_t lse_rows = VARLEN ? static_cast<size_t>(p.total_q) : static_cast<size_t>(T);
      p.lse[(static_cast<size_t>(bc) * p.Hq + h) * lse_rows + qoff + row] = lse;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace prefill
}  // namespace attn

// decode_paged.cuh - one-token attention against a paged KV cache (sm_100a).
//
// The cache layout and the translation follow the page "Snelle
// attention-kernels en operatorfusie versnellen AI-modellen" (the-ai.news),
// section "FlashAttention-type aandacht en gepagineerde aandacht": keys and
// values live in fixed-size physical blocks (16 tokens in the page's vLLM
// example) and a block table maps every logical block of a sequence to a
// physical one; the kernel translates each position through that table.
// The blockwise online softmax of the same section is applied per block.
//
// Work unit (one CTA) = (split, kv-head group, sequence): the logical blocks
// [split*chunk, (split+1)*chunk) of one sequence for KH consecutive kv heads.
//   warps 0..KH-1  consumers, one kv head each, all G = Hq/Hkv query heads of
//                  that kv head at once (the group shares every K/V load)
//   warp  KH       producer: reads the block-table entries of the range and
//                  issues one TMA load per tensor per block (a 3-D view of
//                  the pool brings the 16 token rows of all KH heads at once)
// Per block, a consumer warp computes S^T[16 tokens x 8] = K q^T with
// mma.sync m16n8k16 (query heads padded to 8), updates the running max / sum
// of its heads, transposes P^T into the B-operand layout with movmatrix and
// accumulates O^T[d x 8] += V^T P with ldmatrix.trans-fed mma.sync.  K/V are
// read from HBM exactly once; the tensor-core work per byte is tiny, so the
// kernel is bound by HBM bandwidth.
//
// Output: with one split the bf16 result is written directly; otherwise each
// unit writes its normalised partial output (fp32) and its log-sum-exp, and
// lse_combine merges the splits:  O = sum_i e^{lse_i - M} o_i / sum_i e^{lse_i - M}.
//
// Checks: a sequence length outside [0, max_blocks * 16] is clamped into it
// (the table row holds no more blocks) and a block-table entry outside
// [0, num_blocks) is never loaded: its 16 positions are left out of the
// softmax.  Both set a bit of the device status word.
#pragma once

#include "sm100_ptx.cuh"

namespace attn {
namespace decode {

constexpr int kBlock = 16;   // tokens per physical block
constexpr int kKH = 4;       // kv heads per CTA (consumer warps)
constexpr int kStages = 3;   // K/V blocks in flight per CTA (2 CTAs fit on one SM)

template <int D>
struct Config {
  static constexpr int kChunks = D / 64;                          // 128-byte chunks per head row
  static constexpr uint32_t kChunkBytes = kBlock * 128;           // 16 tokens x 128 B = 2 KB
  static constexpr uint32_t kHeadBytes = kChunks * kChunkBytes;   // one head of one block
};

template <int D>
struct __align__(1024) Smem {
  using C = Config<D>;
  // [stage][head][chunk] -> 16 token rows of 128 B, 128-byte swizzled
  __nv_bfloat16 k[kStages][kKH][C::kChunks][kBlock * 64];
  __nv_bfloat16 v[kStages][kKH][C::kChunks][kBlock * 64];
  uint64_t full[kStages], empty[kStages];
  int bad[kStages];  // 1: the stage's block id lies outside the pool (nothing loaded)
  int abort_flag;
};

template <int D>
constexpr size_t smem_bytes() {
  return sizeof(Smem<D>) + 1024;
}

struct Params {
  const __nv_bfloat16* q;      // [B, Hq, D]
  const int32_t* block_table;  // [B, max_blocks]
  const int32_t* seq_lens;     // [B]
  __nv_bfloat16* o;            // [B, Hq, D]: written by a single split, or null (see part_o)
  float* part_o;               // [num_splits, B, Hq, D]; a single split writes here when o is null
  float* part_lse;             // [num_splits, B, Hq]
  int B, Hq, Hkv, max_blocks;
  int num_blocks;              // pool size: block ids outside [0, num_blocks) are masked
  int num_splits, chunk;       // chunk = blocks per split
  float scale_log2;            // scale * log2(e) (FP8 path: scale * k_scale * log2(e))
  float v_scale = 1.0f;        // FP8 path: V = v_scale * v_cache
};

// Cached tokens of sequence b, clamped to what its table row can name; a
// length outside that range sets kDevStatusBadSeqLen (by one thread, `report`).
__device__ __forceinline__ int checked_len(const int32_t* seq_lens, int b, int max_blocks, bool report) {
  const int L = seq_lens[b];
  const int cap = max_blocks * kBlock;
  if (L >= 0 && L <= cap) return L;
  if (report) atomicOr(&g_devstatus, kDevStatusBadSeqLen);
  return L < 0 ? 0 : cap;
}

// Byte address of token row t, 16-byte unit u of a 128-byte-swizzled chunk.
__device__ __forceinline__ uint32_t sw128(uint32_t chunk_base, int t, int u) {
  return chunk_base + t * 128 + ((u ^ (t & 7)) << 4);
}

template <int D>
__global__ void __launch_bounds__((kKH + 1) * 32, 2)
    paged_decode_split(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const Params p) {
  using C = Config<D>;
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int split = blockIdx.x;
  const int hg = blockIdx.y;  // kv-head group
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kh_act = min(kKH, p.Hkv - hg * kKH);  // kv heads of this group that exist

  // Barrier setup overlaps the previous grid's tail (programmatic launch);
  // global memory is read only after grid_dependency_wait().  Then the
  // combine kernel (this grid's programmatic dependent) may be scheduled; it
  // waits for this grid's completion before it reads any partial.
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kh_act);
    }
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  grid_dependency_wait();
  grid_launch_dependents();

  const int L = checked_len(p.seq_lens, b, p.max_blocks, threadIdx.x == 0 && split == 0 && hg == 0);
  const int nb = (L + kBlock - 1) / kBlock;
  const int blk0 = split * p.chunk;
  const int blk1 = min(nb, blk0 + p.chunk);
  if (blk0 >= blk1) {
    // Empty range.  With several splits the combine skips it (and writes
    // zeros for an empty sequence); with one split this CTA owns the output:
    // O = 0, or a partial o = 0 with lse = -inf.
    if (p.num_splits == 1 && L <= 0) {
      const int G = p.Hq / p.Hkv;
      const int heads = min(kKH, p.Hkv - hg * kKH) * G;
      const size_t head0 = static_cast<size_t>(b) * p.Hq + hg * kKH * G;
      if (p.o != nullptr) {
        __nv_bfloat16* out = p.o + head0 * D;
        for (int i = threadIdx.x; i < heads * D; i += blockDim.x) out[i] = __float2bfloat16_rn(0.f);
      } else {
        for (int i = threadIdx.x; i < heads * D; i += blockDim.x) p.part_o[head0 * D + i] = 0.f;
        for (int i = threadIdx.x; i < heads; i += blockDim.x) p.part_lse[head0 + i] = -INFINITY;
      }
    }
    return;
  }
  const int n = blk1 - blk0;
  __syncthreads();
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == kKH) {
    // ------------------------------ producer ------------------------------
    // Lane i holds block-table entry blk0 + w*32 + i of the current window;
    // lane 0 issues the loads.  Entries past the range are never read.
    const int32_t* row = p.block_table + static_cast<size_t>(b) * p.max_blocks + blk0;
    int issued = 0;
    bool ok = true;
    for (int w = 0; w < n && ok; w += 32) {
      const int mine = (w + lane < n) ? __ldg(row + w + lane) : 0;
      const int cnt = min(32, n - w);
      for (int i = 0; i < cnt; ++i) {
        const int phys = __shfl_sync(0xffffffffu, mine, i);
        const int j = w + i;
        const int s = j % kStages;
        if (lane == 0) {
          ok = mbar_wait(&sm.empty[s], ((j / kStages) & 1) ^ 1, abort_flag);
          if (ok) {
            if (static_cast<unsigned>(phys) < static_cast<unsigned>(p.num_blocks)) {
              // one copy per tensor: the 16 token rows of the group's kKH heads
              // (heads past Hkv are zero-filled and still count as bytes)
              sm.bad[s] = 0;
              mbar_arrive_expect_tx(&sm.full[s], 2 * kKH * C::kHeadBytes);
              tma_load_3d(sm.k[s][0][0], &tmK, &sm.full[s], 0, phys * kBlock, hg * kKH * C::kChunks);
              tma_load_3d(sm.v[s][0][0], &tmV, &sm.full[s], 0, phys * kBlock, hg * kKH * C::kChunks);
            } else {
              // an id outside the pool: nothing is loaded, the consumers skip the block
              sm.bad[s] = 1;
              atomicOr(&g_devstatus, kDevStatusBadBlock);
              mbar_arrive(&sm.full[s]);
            }
            issued = j + 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
    }
    if (lane == 0 && *abort_flag) {
      for (int j = max(0, issued - kStages); j < issued; ++j)
        mbar_wait_drain(&sm.full[j % kStages], (j / kStages) & 1);
    }
    return;
  }

  // ------------------------------- consumers -------------------------------
  if (warp >= kh_act) return;
  const int G = p.Hq / p.Hkv;       // query heads per kv head (<= 8)
  const int hk = hg * kKH + warp;   // kv head of this warp
  const int g_row = lane >> 2;      // B-fragment column (query head) of this lane
  const int quad = lane & 3;

  // q^T as mma B fragments: b0 holds q[g][kk*16 + 2*quad + {0,1}], b1 the same +8.
  uint32_t qf[D / 16][2];
  {
    const bool real = g_row < G;
    const __nv_bfloat16* qrow = p.q + (static_cast<size_t>(b) * p.Hq + hk * G + (real ? g_row : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * quad);
      qf[kk][0] = real ? __ldg(q32) : 0u;
      qf[kk][1] = real ? __ldg(q32 + 4) : 0u;
    }
  }

  float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 domain), heads 2*quad, 2*quad+1
  float l0 = 0.f, l1 = 0.f;              // per-lane partial row sums
  float acc[D / 16][4];
#pragma unroll
  for (int mm = 0; mm < D / 16; ++mm) acc[mm][0] = acc[mm][1] = acc[mm][2] = acc[mm][3] = 0.f;

  const float sl2 = p.scale_log2;
  const int t0 = lane >> 2;  // token rows of this lane in the S^T fragment
  const int t1 = t0 + 8;
  // ldmatrix row addressing: lane provides row (lane & 7) of matrix (lane >> 3)
  const int lm_mat = lane >> 3;
  const int lm_row = lane & 7;

  bool ok = true;
  for (int j = 0; j < n; ++j) {
    const int s = j % kStages;
    ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[s], (j / kStages) & 1, abort_flag));
    if (!ok) break;
    if (sm.bad[s]) {  // a block outside the pool: its keys take no part (warp-uniform)
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
      continue;
    }

    // ---- S^T = K q^T over the 16 tokens of this block ----
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t kbase = smem_u32(sm.k[s][warp][0]);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      // A = K[16 tok x 16 d]: matrices (tok 0-7 | 8-15) x (d 0-7 | 8-15)
      const int t = lm_row + 8 * (lm_mat & 1);
      const int u = (kk & 3) * 2 + (lm_mat >> 1);
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(sw128(kbase + (kk >> 2) * C::kChunkBytes, t, u), a0, a1, a2, a3);
      mma_bf16_16816(sc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
    }
    // ---- mask the tail of the last block ----
    const int pos0 = (blk0 + j) * kBlock;
    const int valid = L - pos0;  // tokens of this block that are in the sequence
    if (t0 >= valid) sc[0] = sc[1] = -INFINITY;
    if (t1 >= valid) sc[2] = sc[3] = -INFINITY;
    if (valid < kBlock) {
      // Slots past the sequence end may hold anything (even NaN); their
      // weight is 0, but 0 * NaN is not 0, so clear this head's V rows.
      uint8_t* vh = reinterpret_cast<uint8_t*>(sm.v[s][warp][0]);
      for (int i = lane; i < (kBlock - valid) * C::kChunks * 8; i += 32) {
        const int unit = i & 7, c = (i >> 3) % C::kChunks, t = valid + (i >> 3) / C::kChunks;
        *reinterpret_cast<uint4*>(vh + c * C::kChunkBytes + t * 128 + unit * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();  // order these writes before the stage's next TMA fill
      __syncwarp();
    }

    // ---- online softmax for the two query heads of this lane ----
    float x0 = fmaxf(sc[0], sc[2]);
    float x1 = fmaxf(sc[1], sc[3]);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, off));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, off));
    }
    const float mn0 = fmaxf(m0, x0 * sl2);  // token 0 of a block is always valid: finite
    const float mn1 = fmaxf(m1, x1 * sl2);
    const float al0 = ex2_approx(m0 - mn0);  // 0 on the first block (m = -inf)
    const float al1 = ex2_approx(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    const float p00 = ex2_approx(fmaf(sc[0], sl2, -mn0));
    const float p01 = ex2_approx(fmaf(sc[1], sl2, -mn1));
    const float p10 = ex2_approx(fmaf(sc[2], sl2, -mn0));
    const float p11 = ex2_approx(fmaf(sc[3], sl2, -mn1));
    l0 = fmaf(l0, al0, p00 + p10);
    l1 = fmaf(l1, al1, p01 + p11);
#pragma unroll
    for (int mm = 0; mm < D / 16; ++mm) {
      acc[mm][0] *= al0;
      acc[mm][1] *= al1;
      acc[mm][2] *= al0;
      acc[mm][3] *= al1;
    }
    // P^T (tokens x heads, C layout) -> P as the k16 x n8 B operand
    const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p00, p01));
    const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p10, p11));

    // ---- O^T[d x 8] += V^T[d x 16 tok] P[16 tok x 8] ----
    const uint32_t vbase = smem_u32(sm.v[s][warp][0]);
#pragma unroll
    for (int mm = 0; mm < D / 16; ++mm) {
      // A = V^T[16 d x 16 tok]: matrices (d 0-7 | 8-15) x (tok 0-7 | 8-15),
      // read transposed from token rows.
      const int t = lm_row + 8 * (lm_mat >> 1);
      const int u = (mm & 3) * 2 + (lm_mat & 1);
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4_trans(sw128(vbase + (mm >> 2) * C::kChunkBytes, t, u), a0, a1, a2, a3);
      mma_bf16_16816(acc[mm], a0, a1, a2, a3, pb0, pb1);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[s]);
  }

  // ---- finish: full row sums, normalise, write ----
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  if (!ok) return;
  // l = 0 only when every block of the range lay outside the pool: O = 0, LSE = -inf
  const float inv0 = l0 > 0.f ? 1.0f / l0 : 0.f, inv1 = l1 > 0.f ? 1.0f / l1 : 0.f;
  const int g0 = 2 * quad, g1 = 2 * quad + 1;
  const size_t head0 = static_cast<size_t>(b) * p.Hq + hk * G;  // first query head of this kv head
  if (p.num_splits == 1 && p.o != nullptr) {
#pragma unroll
    for (int mm = 0; mm < D / 16; ++mm) {
      const int dd = mm * 16 + g_row;
      if (g0 < G) {
        p.o[(head0 + g0) * D + dd] = __float2bfloat16_rn(acc[mm][0] * inv0);
        p.o[(head0 + g0) * D + dd + 8] = __float2bfloat16_rn(acc[mm][2] * inv0);
      }
      if (g1 < G) {
        p.o[(head0 + g1) * D + dd] = __float2bfloat16_rn(acc[mm][1] * inv1);
        p.o[(head0 + g1) * D + dd + 8] = __float2bfloat16_rn(acc[mm][3] * inv1);
      }
    }
  } else {
    const size_t base = static_cast<size_t>(split) * p.B * p.Hq + head0;
#pragma unroll
    for (int mm = 0; mm < D / 16; ++mm) {
      const int dd = mm * 16 + g_row;
      if (g0 < G) {
        p.part_o[(base + g0) * D + dd] = acc[mm][0] * inv0;
        p.part_o[(base + g0) * D + dd + 8] = acc[mm][2] * inv0;
      }
      if (g1 < G) {
        p.part_o[(base + g1) * D + dd] = acc[mm][1] * inv1;
        p.part_o[(base + g1) * D + dd + 8] = acc[mm][3] * inv1;
      }
    }
    if (g_row == 0) {
      constexpr float kLn2 = 0.69314718055994531f;
      if (g0 < G) p.part_lse[base + g0] = (m0 + __log2f(l0)) * kLn2;
      if (g1 < G) p.part_lse[base + g1] = (m1 + __log2f(l1)) * kLn2;
    }
  }
}

// Merge the split partials of every (sequence, query head):
//   M = max_i lse_i,  O = sum_i e^{lse_i - M} o_i / sum_i e^{lse_i - M}.
// WPR warps merge one (sequence, query head) row; a CTA holds
// max(8, WPR) warps, i.e. max(1, 8 / WPR) rows, so that few splits give one
// wave of CTAs and many splits spread each row over up to 32 warps.  Warp w
// of a row takes splits w, w + WPR, ... with a running maximum (no separate
// max pass) and kUnroll rows in flight per lane; lane c owns D/32
// consecutive columns.  The row's warps are merged in shared memory in a
// fixed order (deterministic).  Launched as a programmatic dependent of the
// split kernel: everything before grid_dependency_wait() overlaps its tail.
// kF32: write the merged row as fp32 o [B, Hq, D] plus its natural-log
// lse [B, Hq] (itself a partial that a later merge can take), else as bf16.
// seq_lens null: every one of the num_splits partials of a row is merged
// (partials gathered from other devices; an empty one has lse = -inf).
template <int WPR>
struct CombineShape {
  static constexpr int kWarps = WPR > 8 ? WPR : 8;
  static constexpr int kRows = kWarps / WPR;
};

// One lane's kPer columns of a merged row: tot / ws, and the row's lse from
// its log2-domain maximum M and weight sum ws (ws = 0: no key, o = 0, lse = -inf).
template <int kPer, bool kF32>
__device__ __forceinline__ void store_merged(void* out, float* out_lse, int row_id, int lane, const float* tot,
                                             float M, float ws) {
  constexpr int D = kPer * 32;
  const float inv = ws > 0.f ? 1.0f / ws : 0.f;
  if constexpr (kF32) {
    float* dst = static_cast<float*>(out) + static_cast<size_t>(row_id) * D + lane * kPer;
#pragma unroll
    for (int e = 0; e < kPer; ++e) dst[e] = tot[e] * inv;
    if (lane == 0) out_lse[row_id] = ws > 0.f ? (M + __log2f(ws)) * 0.69314718055994531f : -INFINITY;
  } else {
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(out) + static_cast<size_t>(row_id) * D + lane * kPer;
#pragma unroll
    for (int e = 0; e < kPer; ++e) dst[e] = __float2bfloat16_rn(tot[e] * inv);
  }
}

template <int D, int WPR, bool kF32>
__global__ void __launch_bounds__(CombineShape<WPR>::kWarps * 32)
    lse_combine(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                const int32_t* __restrict__ seq_lens, void* __restrict__ out, float* __restrict__ out_lse, int B,
                int Hq, int num_splits, int chunk, int max_blocks) {
  using Shape = CombineShape<WPR>;
  constexpr int kPer = D / 32;
  constexpr int kUnroll = 8;  // rows in flight per lane: one round for up to 8 splits per warp
  constexpr float kLog2e = 1.4426950408889634f;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int local_row = warp / WPR;
  const int sub = warp % WPR;
  const int row_id = blockIdx.x * Shape::kRows + local_row;  // = b * Hq + h
  const bool live = row_id < B * Hq;
  __shared__ float s_acc[Shape::kWarps][D];
  __shared__ float s_m[Shape::kWarps], s_w[Shape::kWarps];

  grid_dependency_wait();
  grid_launch_dependents();
  int nsp = 0;
  if (live && seq_lens == nullptr) {
    nsp = num_splits;
  } else if (live) {
    const int L = checked_len(seq_lens, row_id / Hq, max_blocks, false);  // the split kernel reports
    nsp = min(num_splits, (((L + kBlock - 1) / kBlock) + chunk - 1) / chunk);  // splits holding data
  }
  const size_t stride = static_cast<size_t>(B) * Hq;  // rows between splits

  float m = -INFINITY, wsum = 0.f;  // log2-domain running max and weight sum
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  for (int i0 = sub; i0 < nsp; i0 += kUnroll * WPR) {
    float lv[kUnroll];
    float ov[kUnroll][kPer];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = i0 + u * WPR;
      const size_t row = static_cast<size_t>(min(i, nsp - 1)) * stride + row_id;
      lv[u] = (i < nsp) ? part_lse[row] * kLog2e : -INFINITY;
      const float* src = part_o + row * D + lane * kPer;
      if constexpr (kPer == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        ov[u][0] = v.x, ov[u][1] = v.y, ov[u][2] = v.z, ov[u][3] = v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        ov[u][0] = v.x, ov[u][1] = v.y;
      }
    }
    float mx = m;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) mx = fmaxf(mx, lv[u]);
    if (mx == -INFINITY) continue;  // no keys in these splits so far (all outside the pool)
    const float sc = ex2_approx(m - mx);  // m = -inf on the first round: 0
    wsum *= sc;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] *= sc;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const float w = ex2_approx(lv[u] - mx);  // 0 for rows past nsp
      wsum += w;
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, ov[u][e], acc[e]);
    }
    m = mx;
  }
  if constexpr (WPR == 1) {
    if (!live) return;
    store_merged<kPer, kF32>(out, out_lse, row_id, lane, acc, m, wsum);  // no key at all: O = 0
    return;
  } else {
#pragma unroll
    for (int e = 0; e < kPer; ++e) s_acc[warp][lane * kPer + e] = acc[e];
    if (lane == 0) {
      s_m[warp] = m;
      s_w[warp] = wsum;
    }
    __syncthreads();
    if (!live || sub != 0) return;
    // the first warp of the row merges its WPR warps
    const int w0 = local_row * WPR;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WPR; ++w) M = fmaxf(M, s_m[w0 + w]);
    float ws = 0.f;
    float tot[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) tot[e] = 0.f;
    if (M != -INFINITY) {  // else: empty sequence, or no key inside the pool: O = 0
#pragma unroll
      for (int w = 0; w < WPR; ++w) {
        const float f = ex2_approx(s_m[w0 + w] - M);  // warps without rows: -inf -> 0
        ws = fmaf(f, s_w[w0 + w], ws);
#pragma unroll
        for (int e = 0; e < kPer; ++e) tot[e] = fmaf(f, s_acc[w0 + w][lane * kPer + e], tot[e]);
      }
    }
    store_merged<kPer, kF32>(out, out_lse, row_id, lane, tot, M, ws);
  }
}

}  // namespace decode
}  // namespace attn

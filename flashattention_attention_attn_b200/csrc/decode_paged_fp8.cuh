// decode_paged_fp8.cuh - one-token attention against a paged KV cache whose
// keys and values are stored as FP8 e4m3 with one scale per tensor
// (K = k_scale * k_cache, V = v_scale * v_cache), head dim 128.
//
// Same work decomposition as paged_decode_split (decode_paged.cuh): one CTA
// per (split, group of kKH kv heads, sequence); a producer warp reads the
// block table and issues one TMA per tensor per 16-token block, covering the
// group's kKH heads (a head row of e4m3 is exactly one 128-byte swizzle
// row); one consumer warp per kv head serves all G = Hq/Hkv query heads of
// that kv head.
//
// Scores: S^T[16 tokens x 8 heads] = K q^T with f16 mma.sync.  ldmatrix on
// the e4m3 tile gives each lane 4 consecutive bytes (head-dim columns
// 4q..4q+3 of one token); cvt.rn.f16x2.e4m3x2 turns them into two f16
// pairs.  Those pairs fill the A fragment in a permuted order of the head
// dimension, and q is laid into the B fragment with the same permutation:
// a dot product does not depend on the order of its terms.  q carries
// scale * k_scale * log2(e), so the scores come out in the log2 domain.
// Output: O^T[d x 8 heads] += V^T P, with P (transposed by movmatrix) as the
// B operand.  ldmatrix.trans on the e4m3 tile gives each lane two tokens x
// two adjacent columns (2j, 2j+1); byte permutes split them into an f16 pair
// over the two tokens for column 2j and one for column 2j+1, which become
// the A-fragment rows j and j + 8: each 16-row output tile holds its 16
// columns in the order (0, 2, .., 14, 1, 3, .., 15).  v_scale is applied
// once at the end.  Sequence lengths and block ids are checked as in
// paged_decode_split.
#pragma once

#include "decode_paged.cuh"
#include "sm100_ptx.cuh"

namespace attn {
namespace decode {

// Stages in flight and resident CTAs per SM.  5 x 16 KB per CTA measured
// best: 82% vs 78% of the HBM copy peak with 6 on long_decode_131k, equal on
// paged_decode_b64; 4 stages with 3 CTAs or 3 with 4 gained nothing.
constexpr int kFp8Stages = 5;     // 16 KB per stage (K + V of 4 heads)
constexpr int kFp8CtasPerSm = 2;  // resident CTAs per SM
constexpr int kFp8D = 128;      // head dim served by the FP8 path
constexpr uint32_t kFp8HeadBytes = kBlock * kFp8D;  // one head of one block: 16 rows x 128 B

struct __align__(1024) SmemFp8 {
  uint8_t k[kFp8Stages][kKH][kFp8HeadBytes];
  uint8_t v[kFp8Stages][kKH][kFp8HeadBytes];
  uint64_t full[kFp8Stages], empty[kFp8Stages];
  int bad[kFp8Stages];  // 1: the stage's block id lies outside the pool (nothing loaded)
  int abort_flag;
};

constexpr size_t smem_bytes_fp8() { return sizeof(SmemFp8) + 1024; }

__global__ void __launch_bounds__((kKH + 1) * 32, kFp8CtasPerSm)
    paged_decode_split_fp8(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const Params p) {
  constexpr int D = kFp8D;
  extern __shared__ uint8_t smem_raw[];
  SmemFp8& sm = *reinterpret_cast<SmemFp8*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int split = blockIdx.x;
  const int hg = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kh_act = min(kKH, p.Hkv - hg * kKH);

  // As in the bf16 kernel: barrier setup before the wait for the previous
  // grid, global reads after it, then the combine may be scheduled.
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFp8Stages; ++s) {
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
  const int G = p.Hq / p.Hkv;
  if (blk0 >= blk1) {
    if (p.num_splits == 1 && L <= 0) {
      const int heads = min(kKH, p.Hkv - hg * kKH) * G;
      __nv_bfloat16* out = p.o + (static_cast<size_t>(b) * p.Hq + hg * kKH * G) * D;
      for (int i = threadIdx.x; i < heads * D; i += blockDim.x) out[i] = __float2bfloat16_rn(0.f);
    }
    return;
  }
  const int n = blk1 - blk0;
  __syncthreads();
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == kKH) {
    // ------------------------------ producer ------------------------------
    const int32_t* row = p.block_table + static_cast<size_t>(b) * p.max_blocks + blk0;
    int issued = 0;
    bool ok = true;
    for (int w = 0; w < n && ok; w += 32) {
      const int mine = (w + lane < n) ? __ldg(row + w + lane) : 0;
      const int cnt = min(32, n - w);
      for (int i = 0; i < cnt; ++i) {
        const int phys = __shfl_sync(0xffffffffu, mine, i);
        const int j = w + i;
        const int s = j % kFp8Stages;
        if (lane == 0) {
          ok = mbar_wait(&sm.empty[s], ((j / kFp8Stages) & 1) ^ 1, abort_flag);
          if (ok) {
            if (static_cast<unsigned>(phys) < static_cast<unsigned>(p.num_blocks)) {
              // one copy per tensor: the 16 token rows of the group's kKH heads
              // (heads past Hkv are zero-filled and still count as bytes)
              sm.bad[s] = 0;
              mbar_arrive_expect_tx(&sm.full[s], 2 * kKH * kFp8HeadBytes);
              tma_load_3d(sm.k[s][0], &tmK, &sm.full[s], 0, phys * kBlock, hg * kKH);
              tma_load_3d(sm.v[s][0], &tmV, &sm.full[s], 0, phys * kBlock, hg * kKH);
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
      for (int j = max(0, issued - kFp8Stages); j < issued; ++j)
        mbar_wait_drain(&sm.full[j % kFp8Stages], (j / kFp8Stages) & 1);
    }
    return;
  }

  // ------------------------------- consumers -------------------------------
  if (warp >= kh_act) return;
  const int hk = hg * kKH + warp;
  const int g_row = lane >> 2;  // query head of this lane in B fragments / O rows
  const int quad = lane & 3;
  const bool real_row = g_row < G;

  // q^T as f16 B fragments, head dim permuted as the K fragments are:
  // for column group kg (32 columns) and half hf, b0 = q[4*quad + {0,1}],
  // b1 = q[4*quad + {2,3}] of columns 32*kg + 16*hf.
  uint32_t qf[D / 32][2][2];
  {
    const __nv_bfloat16* qrow = p.q + (static_cast<size_t>(b) * p.Hq + hk * G + (real_row ? g_row : 0)) * D;
    const float c = p.scale_log2;  // scale * k_scale * log2(e)
#pragma unroll
    for (int kg = 0; kg < D / 32; ++kg)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const uint2 raw = real_row ? __ldg(reinterpret_cast<const uint2*>(qrow + 32 * kg + 16 * hf + 4 * quad))
                                   : make_uint2(0u, 0u);
        const float q0 = __uint_as_float(raw.x << 16), q1 = __uint_as_float(raw.x & 0xffff0000u);
        const float q2 = __uint_as_float(raw.y << 16), q3 = __uint_as_float(raw.y & 0xffff0000u);
        qf[kg][hf][0] = pack_f16x2(q0 * c, q1 * c);
        qf[kg][hf][1] = pack_f16x2(q2 * c, q3 * c);
      }
  }

  float m0 = -INFINITY, m1 = -INFINITY;  // running max, heads 2*quad, 2*quad+1 (log2 domain)
  float l0 = 0.f, l1 = 0.f;
  // O^T tile u: acc[u][0] = O[2q][16u + 2j], acc[u][1] = O[2q+1][16u + 2j],
  // acc[u][2] = O[2q][16u + 2j + 1], acc[u][3] = O[2q+1][16u + 2j + 1]; j = lane / 4
  float acc[D / 16][4];
#pragma unroll
  for (int u = 0; u < D / 16; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;

  const int t0 = lane >> 2, t1 = t0 + 8;
  const int lm_mat = lane >> 3, lm_row = lane & 7;
  bool ok = true;
  for (int j = 0; j < n; ++j) {
    const int s = j % kFp8Stages;
    ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[s], (j / kFp8Stages) & 1, abort_flag));
    if (!ok) break;
    if (sm.bad[s]) {  // a block outside the pool: its keys take no part (warp-uniform)
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
      continue;
    }

    // ---- S^T = K q^T (log2 domain) ----
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t kbase = smem_u32(sm.k[s][warp]);
#pragma unroll
    for (int kg = 0; kg < D / 32; ++kg) {
      const int t = lm_row + 8 * (lm_mat & 1);
      const int u = 2 * kg + (lm_mat >> 1);
      uint32_t r0, r1, r2, r3;
      ldmatrix_x4(sw128(kbase, t, u), r0, r1, r2, r3);
      mma_f16_16816(sc, e4m3x2_to_f16x2(r0 & 0xffffu), e4m3x2_to_f16x2(r1 & 0xffffu), e4m3x2_to_f16x2(r0 >> 16),
                    e4m3x2_to_f16x2(r1 >> 16), qf[kg][0][0], qf[kg][0][1]);
      mma_f16_16816(sc, e4m3x2_to_f16x2(r2 & 0xffffu), e4m3x2_to_f16x2(r3 & 0xffffu), e4m3x2_to_f16x2(r2 >> 16),
                    e4m3x2_to_f16x2(r3 >> 16), qf[kg][1][0], qf[kg][1][1]);
    }
    const int pos0 = (blk0 + j) * kBlock;
    const int valid = L - pos0;
    if (t0 >= valid) sc[0] = sc[1] = -INFINITY;
    if (t1 >= valid) sc[2] = sc[3] = -INFINITY;
    if (valid < kBlock) {
      // slots past the sequence end may hold anything (e4m3 NaN included): clear V rows
      uint8_t* vh = sm.v[s][warp];
      for (int i = lane; i < (kBlock - valid) * 8; i += 32)
        *reinterpret_cast<uint4*>(vh + (valid + (i >> 3)) * 128 + (i & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();
      __syncwarp();
    }

    // ---- online softmax (heads 2*quad, 2*quad+1 of this lane) ----
    float x0 = fmaxf(sc[0], sc[2]);
    float x1 = fmaxf(sc[1], sc[3]);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, off));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, off));
    }
    const float mn0 = fmaxf(m0, x0), mn1 = fmaxf(m1, x1);
    const float al0 = ex2_approx(m0 - mn0), al1 = ex2_approx(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    const float p00 = ex2_approx(sc[0] - mn0), p01 = ex2_approx(sc[1] - mn1);
    const float p10 = ex2_approx(sc[2] - mn0), p11 = ex2_approx(sc[3] - mn1);
    l0 = fmaf(l0, al0, p00 + p10);
    l1 = fmaf(l1, al1, p01 + p11);
#pragma unroll
    for (int u = 0; u < D / 16; ++u) {
      acc[u][0] *= al0;
      acc[u][1] *= al1;
      acc[u][2] *= al0;
      acc[u][3] *= al1;
    }
    // P^T (tokens x heads, C layout) -> P as the k16 x n8 B operand
    const uint32_t pb0 = movmatrix_trans(pack_f16x2(p00, p01));
    const uint32_t pb1 = movmatrix_trans(pack_f16x2(p10, p11));

    // ---- O^T[d x 8] += V^T P ----
    const uint32_t vbase = smem_u32(sm.v[s][warp]);
#pragma unroll
    for (int ux = 0; ux < D / 32; ++ux) {
      const int t = lm_row + 8 * (lm_mat & 1);
      const int u = 2 * ux + (lm_mat >> 1);
      uint32_t r[4];
      ldmatrix_x4_trans(sw128(vbase, t, u), r[0], r[1], r[2], r[3]);
      // r[0]/r[1]: tokens 0-7 / 8-15 of unit 2ux; r[2]/r[3]: the same of unit 2ux+1.
      // Lane bytes: {V[2q][2j], V[2q][2j+1], V[2q+1][2j], V[2q+1][2j+1]}, j = lane / 4.
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const uint32_t lo = r[2 * h2], hi = r[2 * h2 + 1];
        const uint32_t a0 = e4m3x2_to_f16x2(prmt(lo, 0u, 0x20u));  // column 2j, tokens 2q, 2q+1
        const uint32_t a1 = e4m3x2_to_f16x2(prmt(lo, 0u, 0x31u));  // column 2j + 1
        const uint32_t a2 = e4m3x2_to_f16x2(prmt(hi, 0u, 0x20u));  // column 2j, tokens 8 + ...
        const uint32_t a3 = e4m3x2_to_f16x2(prmt(hi, 0u, 0x31u));
        mma_f16_16816(acc[2 * ux + h2], a0, a1, a2, a3, pb0, pb1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[s]);
  }

#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  if (!ok) return;
  const int g0 = 2 * quad, g1 = 2 * quad + 1;
  // l = 0 only when every block of the range lay outside the pool: O = 0, LSE = -inf
  const float inv0 = l0 > 0.f ? p.v_scale / l0 : 0.f, inv1 = l1 > 0.f ? p.v_scale / l1 : 0.f;
  const int j2 = 2 * g_row;  // this lane's even column within each 16-column tile
  const size_t head0 = static_cast<size_t>(b) * p.Hq + hk * G;
  if (p.num_splits == 1) {
#pragma unroll
    for (int u = 0; u < D / 16; ++u) {
      if (g0 < G)
        *reinterpret_cast<uint32_t*>(p.o + (head0 + g0) * D + 16 * u + j2) =
            pack_bf16x2(acc[u][0] * inv0, acc[u][2] * inv0);
      if (g1 < G)
        *reinterpret_cast<uint32_t*>(p.o + (head0 + g1) * D + 16 * u + j2) =
            pack_bf16x2(acc[u][1] * inv1, acc[u][3] * inv1);
    }
  } else {
    const size_t base = static_cast<size_t>(split) * p.B * p.Hq + head0;
#pragma unroll
    for (int u = 0; u < D / 16; ++u) {
      if (g0 < G)
        *reinterpret_cast<float2*>(p.part_o + (base + g0) * D + 16 * u + j2) =
            make_float2(acc[u][0] * inv0, acc[u][2] * inv0);
      if (g1 < G)
        *reinterpret_cast<float2*>(p.part_o + (base + g1) * D + 16 * u + j2) =
            make_float2(acc[u][1] * inv1, acc[u][3] * inv1);
    }
    if (g_row == 0) {
      constexpr float kLn2 = 0.69314718055994531f;
      if (g0 < G) p.part_lse[base + g0] = (m0 + __log2f(l0)) * kLn2;
      if (g1 < G) p.part_lse[base + g1] = (m1 + __log2f(l1)) * kLn2;
    }
  }
}

}  // namespace decode
}  // namespace attn

// attn_api.cu - host side of the C ABI declared in include/attn.h: argument
// validation, TMA descriptor construction, launch configuration and the
// stream-ordered workspace of the split-KV decode.  Every step of the
// computation runs in the kernels included below; there is no CPU path.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "decode_paged.cuh"
#include "decode_paged_fp8.cuh"
#include "prefill_sm100.cuh"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kMaxDevices = 64;

__global__ void fill_no_keys(__nv_bfloat16* o, float* lse, size_t n_o, size_t n_lse) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t k = i; k < n_o; k += stride) o[k] = __float2bfloat16_rn(0.f);
  if (lse != nullptr)
    for (size_t k = i; k < n_lse; k += stride) lse[k] = -INFINITY;
}

struct DeviceState {
  bool probed = false;
  int status = ATTN_ERR_CUDA;  // result of the support check
  int sms = 0;
  bool attrs_set = false;
  cudaMemPool_t pool = nullptr;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// The prefill kernels move registers from warpgroup 2 to the softmax
// warpgroups with setmaxnreg; the increase waits until the launch's
// allocation can supply it, so every prefill kernel must have been compiled
// with the per-thread count the split was sized for.  Checked once per
// device, before any prefill is launched.
bool prefill_registers_fit() {
  const void* fns[] = {
      reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<64, prefill::kDense>),
      reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<128, prefill::kDense>),
      reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<64, prefill::kVarlen>),
      reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<128, prefill::kVarlen>),
      reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<64, prefill::kPaged>),
      reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<128, prefill::kPaged>),
  };
  for (const void* fn : fns) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    const long long have = static_cast<long long>(fa.numRegs) * prefill::kThreads;
    const long long need = 2LL * 128 * prefill::kSoftmaxRegs + 128LL * prefill::kOtherRegs;
    if (have < need) return false;
  }
  return true;
}

// Probe a device once: sm_100 (compute capability 10.0) and a loadable image.
int probe_device(int dev, DeviceState** out) {
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& st = g_dev[dev];
  if (!st.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      st.status = ATTN_ERR_CUDA;
    } else if (major != 10 || minor != 0) {
      st.status = ATTN_ERR_UNSUPPORTED;
    } else {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, prefill::prefill_fwd_sm100<128, prefill::kDense>) != cudaSuccess) {
        cudaGetLastError();
        st.status = ATTN_ERR_UNSUPPORTED;  // no sm_100a image for this device
      } else if (!prefill_registers_fit()) {
        st.status = ATTN_ERR_UNSUPPORTED;  // the prefill's register split would not fit its launch
      } else if (encode_tiled() == nullptr) {
        st.status = ATTN_ERR_CUDA;
      } else {
        st.status = ATTN_OK;
      }
    }
    st.sms = sms;
    st.probed = true;
  }
  *out = &st;
  return st.status;
}

// Per-device one-time launch set-up (dynamic shared memory limits, pool).
int prepare_device(int dev, DeviceState* st) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (st->attrs_set) return ATTN_OK;
  const struct {
    const void* fn;
    size_t bytes;
  } kernels[] = {
      {reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<64, prefill::kDense>), prefill::smem_bytes<64>()},
      {reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<128, prefill::kDense>), prefill::smem_bytes<128>()},
      {reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<64, prefill::kVarlen>), prefill::smem_bytes<64>()},
      {reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<128, prefill::kVarlen>), prefill::smem_bytes<128>()},
      {reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<64, prefill::kPaged>), prefill::smem_bytes<64>()},
      {reinterpret_cast<const void*>(prefill::prefill_fwd_sm100<128, prefill::kPaged>), prefill::smem_bytes<128>()},
      {reinterpret_cast<const void*>(decode::paged_decode_split<64>), decode::smem_bytes<64>()},
      {reinterpret_cast<const void*>(decode::paged_decode_split<128>), decode::smem_bytes<128>()},
      {reinterpret_cast<const void*>(decode::paged_decode_split_fp8), decode::smem_bytes_fp8()},
  };
  for (const auto& k : kernels)
    if (cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(k.bytes)) !=
        cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
  cudaMemPoolProps props;
  std::memset(&props, 0, sizeof(props));
  props.allocType = cudaMemAllocationTypePinned;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  if (cudaMemPoolCreate(&st->pool, &props) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  uint64_t keep = UINT64_MAX;  // keep freed workspace cached in the pool
  cudaMemPoolSetAttribute(st->pool, cudaMemPoolAttrReleaseThreshold, &keep);
  st->attrs_set = true;
  return ATTN_OK;
}

int current_device_state(DeviceState** st) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  int rc = probe_device(dev, st);
  if (rc != ATTN_OK) return rc;
  return prepare_device(dev, *st);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 4-D bf16 map over a [B, rows, H, D] tensor: dims (D, H, rows, B),
// box (64, 1, 128, 1), 128-byte swizzle.
int make_map_bthd(CUtensorMap* map, const void* base, int B, int rows, int H, int D) {
  cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(rows), cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(D) * 2, cuuint64_t(H) * D * 2, cuuint64_t(rows) * H * D * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode_tiled()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 2-D bf16 map over a paged pool of num_blocks 16-token blocks seen as
// [tokens, Hkv * D]: box (64, 16).  When the caller does not give the pool
// size, num_blocks is kMaxPoolBlocks (the largest count int32 token
// coordinates address); the kernels load only ids below num_blocks.
int make_map_pool(CUtensorMap* map, const void* base, int Hkv, int D, int num_blocks) {
  const cuuint64_t tokens = cuuint64_t(num_blocks) * decode::kBlock;
  cuuint64_t dims[2] = {cuuint64_t(Hkv) * D, tokens};
  cuuint64_t strides[1] = {cuuint64_t(Hkv) * D * 2};
  cuuint32_t box[2] = {64, 16};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode_tiled()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 3-D map over a paged pool for the decode kernels: dims (one 128-byte row
// of a head, tokens, 128-byte rows of a token), i.e. the token stride is
// listed before the smaller row stride, so that one box of
// (row, 16 tokens, rows_per_group) lands in shared memory as
// [row of the group][token][128 bytes] -- one copy per tensor and block.
int make_map_pool_group(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes,
                        int rows_per_token, int rows_per_group, int num_blocks) {
  const cuuint64_t tokens = cuuint64_t(num_blocks) * decode::kBlock;
  const cuuint32_t row_elems = 128 / elem_bytes;
  cuuint64_t dims[3] = {row_elems, tokens, cuuint64_t(rows_per_token)};
  cuuint64_t strides[2] = {cuuint64_t(rows_per_token) * 128, 128};
  cuuint32_t box[3] = {row_elems, 16, cuuint32_t(rows_per_group)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode_tiled()(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

int make_map_decode_bf16(CUtensorMap* map, const void* base, int Hkv, int D, int num_blocks) {
  return make_map_pool_group(map, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Hkv * D / 64, decode::kKH * D / 64,
                             num_blocks);
}

int make_map_decode_fp8(CUtensorMap* map, const void* base, int Hkv, int num_blocks) {
  return make_map_pool_group(map, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Hkv, decode::kKH, num_blocks);
}

int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Launch as a programmatic dependent of the previous work on the stream: the
// CTAs may be scheduled during the previous grid's tail and do their setup
// there; every kernel launched this way calls grid_dependency_wait() before
// its first global memory access.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
               Args&&... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

template <int D>
int launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                   int T, int S, int causal, float scale, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (make_map_bthd(&mq, q, B, T, Hq, D) || make_map_bthd(&mk, k, B, S, Hkv, D) ||
      make_map_bthd(&mv, v, B, S, Hkv, D))
    return ATTN_ERR_CUDA;
  prefill::Params p;
  std::memset(&p, 0, sizeof(p));
  p.lse = lse;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.T = T;
  p.S = S;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_mblocks = (T + 2 * prefill::kBM - 1) / (2 * prefill::kBM);
  const long long grid = static_cast<long long>(p.num_mblocks) * Hq * B;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  return launch_pdl(prefill::prefill_fwd_sm100<D, prefill::kDense>, dim3(static_cast<unsigned>(grid)),
                    dim3(prefill::kThreads), prefill::smem_bytes<D>(), stream, mq, mk, mv, p);
}

// Packed batches of up to 32 sequences launch one CTA per (head, work item),
// a work item being one 256-row query block of one sequence.  A sequence of
// l rows has ceil(l / 256) of them, so at most (total_q + 255 B) / 256 exist
// (at least 1 here: B, total_q >= 1); CTAs past the last one return at once.
// Larger batches (0) take the full grid of ceil(max_seqlen_q / 256) blocks
// for every (sequence, head), where CTAs past a sequence's end exit at once.
int compact_items(int B, int num_mblocks, int total_q) {
  if (B > 32) return 0;
  const long long full = static_cast<long long>(num_mblocks) * B;
  const long long bound = (static_cast<long long>(total_q) + static_cast<long long>(B) * (2 * prefill::kBM - 1)) /
                          (2 * prefill::kBM);
  return static_cast<int>(bound < full ? bound : full);
}

// Packed sequences: the maps see [total, H, D] as one batch.
template <int D>
int launch_prefill_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* cu_q,
                          const int32_t* cu_k, int B, int max_q, int total_q, int total_k, int Hq, int Hkv,
                          int causal, float scale, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (make_map_bthd(&mq, q, 1, total_q, Hq, D) || make_map_bthd(&mk, k, 1, total_k, Hkv, D) ||
      make_map_bthd(&mv, v, 1, total_k, Hkv, D))
    return ATTN_ERR_CUDA;
  prefill::Params p;
  std::memset(&p, 0, sizeof(p));
  p.lse = lse;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.T = max_q;
  p.S = 0;
  p.total_q = total_q;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_mblocks = (max_q + 2 * prefill::kBM - 1) / (2 * prefill::kBM);
  p.items = compact_items(B, p.num_mblocks, total_q);
  const long long grid = static_cast<long long>(p.items > 0 ? p.items : static_cast<long long>(p.num_mblocks) * B) * Hq;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  return launch_pdl(prefill::prefill_fwd_sm100<D, prefill::kVarlen>, dim3(static_cast<unsigned>(grid)),
                    dim3(prefill::kThreads), prefill::smem_bytes<D>(), stream, mq, mk, mv, p);
}

// Chunked prefill against the paged cache: packed queries as in varlen,
// keys and values gathered through the block table from the pool maps.
template <int D>
int launch_prefill_paged(const void* q, const void* kc, const void* vc, const int32_t* table, const int32_t* lens,
                         const int32_t* cu_q, void* o, float* lse, int B, int max_q, int total_q, int Hq, int Hkv,
                         int max_blocks, int num_blocks, int causal, float scale, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (make_map_bthd(&mq, q, 1, total_q, Hq, D) || make_map_pool(&mk, kc, Hkv, D, num_blocks) ||
      make_map_pool(&mv, vc, Hkv, D, num_blocks))
    return ATTN_ERR_CUDA;
  prefill::Params p;
  std::memset(&p, 0, sizeof(p));
  p.lse = lse;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.cu_q = cu_q;
  p.block_table = table;
  p.seq_lens = lens;
  p.max_blocks = max_blocks;
  p.num_blocks = num_blocks;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.T = max_q;
  p.total_q = total_q;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_mblocks = (max_q + 2 * prefill::kBM - 1) / (2 * prefill::kBM);
  p.items = compact_items(B, p.num_mblocks, total_q);
  const long long grid = static_cast<long long>(p.items > 0 ? p.items : static_cast<long long>(p.num_mblocks) * B) * Hq;
  if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  return launch_pdl(prefill::prefill_fwd_sm100<D, prefill::kPaged>, dim3(static_cast<unsigned>(grid)),
                    dim3(prefill::kThreads), prefill::smem_bytes<D>(), stream, mq, mk, mv, p);
}

// Splits for num_splits <= 0.  The host does not know the sequence lengths
// (they are on the device), so the choice assumes every sequence fills
// max_blocks: a single sequence is cut into one wave of equal units
// (ctas_per_sm decode CTAs fit on an SM); a batch into about three waves, so
// that the scheduler can balance units of unequal length.  (A sweep on a
// batch of 64 sequences of 256-4096 tokens put three waves -- 7 splits --
// ahead of four -- 10 splits -- for both caches, and two far behind.)  At
// least 8 blocks per unit.
int auto_splits(int B, int groups, int max_blocks, int sms, int ctas_per_sm = 2) {
  const long long slots = static_cast<long long>(ctas_per_sm) * sms;
  const long long waves = (B == 1) ? 1 : 3;
  const long long blocks = static_cast<long long>(B) * groups * max_blocks;
  long long chunk = (blocks + waves * slots - 1) / (waves * slots);
  if (chunk < 8) chunk = 8;
  if (chunk > max_blocks) chunk = max_blocks;
  return static_cast<int>((max_blocks + chunk - 1) / chunk);
}

// The LSE merge, launched as a programmatic dependent of the split kernel so
// that its launch and prologue overlap the split kernel's tail.  WPR warps
// per (sequence, head) row: about 8 splits per warp, at most 32 warps.
template <int D, int WPR, bool kF32>
int launch_combine_wpr(const decode::Params& p, const int32_t* lens, void* out, float* out_lse,
                       cudaStream_t stream) {
  using Shape = decode::CombineShape<WPR>;
  const long long rows = static_cast<long long>(p.B) * p.Hq;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>((rows + Shape::kRows - 1) / Shape::kRows), 1, 1);
  cfg.blockDim = dim3(Shape::kWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float* po = p.part_o;
  const float* pl = p.part_lse;
  if (cudaLaunchKernelEx(&cfg, decode::lse_combine<D, WPR, kF32>, po, pl, lens, out, out_lse, p.B, p.Hq,
                         p.num_splits, p.chunk, p.max_blocks) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// Merge p.num_splits partials per row into out: bf16 O, or (kF32) fp32 o
// plus out_lse.  lens null: every partial of a row is merged.
template <int D, bool kF32 = false>
int launch_combine(const decode::Params& p, const int32_t* lens, void* out, float* out_lse, cudaStream_t stream) {
  const int per_warp = 8;
  const int need = (p.num_splits + per_warp - 1) / per_warp;
  if (need <= 1) return launch_combine_wpr<D, 1, kF32>(p, lens, out, out_lse, stream);
  if (need <= 2) return launch_combine_wpr<D, 2, kF32>(p, lens, out, out_lse, stream);
  if (need <= 4) return launch_combine_wpr<D, 4, kF32>(p, lens, out, out_lse, stream);
  if (need <= 8) return launch_combine_wpr<D, 8, kF32>(p, lens, out, out_lse, stream);
  if (need <= 16) return launch_combine_wpr<D, 16, kF32>(p, lens, out, out_lse, stream);
  return launch_combine_wpr<D, 32, kF32>(p, lens, out, out_lse, stream);
}

// o_part / lse_part non-null: the result is the partial (fp32 o [B, Hq, D],
// natural-log lse [B, Hq]) over the keys this call sees, o unused.
template <int D>
int launch_decode(const void* q, const void* kc, const void* vc, const int32_t* table, const int32_t* lens, int B,
                  int Hq, int Hkv, int max_blocks, int num_blocks, int num_splits, void* o, cudaStream_t stream,
                  const DeviceState* st, float* o_part = nullptr, float* lse_part = nullptr) {
  CUtensorMap mk, mv;
  if (make_map_decode_bf16(&mk, kc, Hkv, D, num_blocks) || make_map_decode_bf16(&mv, vc, Hkv, D, num_blocks))
    return ATTN_ERR_CUDA;
  const int groups = (Hkv + decode::kKH - 1) / decode::kKH;
  if (num_splits <= 0) num_splits = auto_splits(B, groups, max_blocks, st->sms);
  if (num_splits > max_blocks) num_splits = max_blocks;
  const int chunk = (max_blocks + num_splits - 1) / num_splits;
  num_splits = (max_blocks + chunk - 1) / chunk;  // drop splits that can never hold a block
  if (num_splits > 65535 || groups > 65535 || B > 65535) return ATTN_ERR_UNSUPPORTED;

  decode::Params p;
  const bool partial = o_part != nullptr;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.block_table = table;
  p.seq_lens = lens;
  p.o = partial ? nullptr : static_cast<__nv_bfloat16*>(o);
  p.part_o = (partial && num_splits == 1) ? o_part : nullptr;  // a single split writes the partial itself
  p.part_lse = (partial && num_splits == 1) ? lse_part : nullptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.max_blocks = max_blocks;
  p.num_blocks = num_blocks;
  p.num_splits = num_splits;
  p.chunk = chunk;
  p.scale_log2 = (1.0f / std::sqrt(static_cast<float>(D))) * 1.4426950408889634f;

  void* ws = nullptr;
  if (num_splits > 1) {
    const size_t rows = static_cast<size_t>(num_splits) * B * Hq;
    const size_t bytes = rows * D * sizeof(float) + rows * sizeof(float);
    // Outside capture the workspace comes from the library's pool; inside a
    // stream capture from cudaMallocAsync, which becomes a graph memory node.
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    const cudaError_t ae = (cap == cudaStreamCaptureStatusActive)
                               ? cudaMallocAsync(&ws, bytes, stream)
                               : cudaMallocFromPoolAsync(&ws, bytes, st->pool, stream);
    if (ae != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    p.part_o = static_cast<float*>(ws);
    p.part_lse = p.part_o + rows * D;
  }
  dim3 grid(num_splits, groups, B);
  int rc = launch_pdl(decode::paged_decode_split<D>, grid, dim3((decode::kKH + 1) * 32), decode::smem_bytes<D>(),
                      stream, mk, mv, p);
  if (rc == ATTN_OK && num_splits > 1)
    rc = partial ? launch_combine<D, true>(p, lens, o_part, lse_part, stream)
                 : launch_combine<D>(p, lens, o, nullptr, stream);
  if (ws != nullptr) cudaFreeAsync(ws, stream);
  return rc;
}

// FP8 (e4m3) cache: the same split / combine structure, 128-dim heads.
int launch_decode_fp8(const void* q, const void* kc, const void* vc, const int32_t* table, const int32_t* lens,
                      int B, int Hq, int Hkv, int max_blocks, int num_blocks, int num_splits, float k_scale,
                      float v_scale, void* o, cudaStream_t stream, const DeviceState* st) {
  constexpr int D = decode::kFp8D;
  CUtensorMap mk, mv;
  if (make_map_decode_fp8(&mk, kc, Hkv, num_blocks) || make_map_decode_fp8(&mv, vc, Hkv, num_blocks))
    return ATTN_ERR_CUDA;
  const int groups = (Hkv + decode::kKH - 1) / decode::kKH;
  if (num_splits <= 0) num_splits = auto_splits(B, groups, max_blocks, st->sms, decode::kFp8CtasPerSm);
  if (num_splits > max_blocks) num_splits = max_blocks;
  const int chunk = (max_blocks + num_splits - 1) / num_splits;
  num_splits = (max_blocks + chunk - 1) / chunk;
  if (num_splits > 65535 || groups > 65535 || B > 65535) return ATTN_ERR_UNSUPPORTED;
  decode::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.block_table = table;
  p.seq_lens = lens;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.part_o = nullptr;
  p.part_lse = nullptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.max_blocks = max_blocks;
  p.num_blocks = num_blocks;
  p.num_splits = num_splits;
  p.chunk = chunk;
  p.scale_log2 = (1.0f / std::sqrt(static_cast<float>(D))) * k_scale * 1.4426950408889634f;
  p.v_scale = v_scale;
  void* ws = nullptr;
  if (num_splits > 1) {
    const size_t rows = static_cast<size_t>(num_splits) * B * Hq;
    const size_t bytes = rows * D * sizeof(float) + rows * sizeof(float);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    const cudaError_t ae = (cap == cudaStreamCaptureStatusActive)
                               ? cudaMallocAsync(&ws, bytes, stream)
                               : cudaMallocFromPoolAsync(&ws, bytes, st->pool, stream);
    if (ae != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    p.part_o = static_cast<float*>(ws);
    p.part_lse = p.part_o + rows * D;
  }
  dim3 grid(num_splits, groups, B);
  int rc = launch_pdl(decode::paged_decode_split_fp8, grid, dim3((decode::kKH + 1) * 32), decode::smem_bytes_fp8(),
                      stream, mk, mv, p);
  if (rc == ATTN_OK && num_splits > 1) rc = launch_combine<D>(p, lens, o, nullptr, stream);
  if (ws != nullptr) cudaFreeAsync(ws, stream);
  return rc;
}

}  // namespace
}  // namespace attn

using namespace attn;

namespace attn {
namespace {

// Host checks shared by the paged entry points.  num_blocks: the pool size
// given by the caller (checked entry points) or kMaxPoolBlocks.
int check_paged_common(int B, int Hq, int Hkv, int d, int block_size, int max_blocks, int num_blocks) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || block_size <= 0) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (B == 0) return ATTN_OK;
  if (max_blocks <= 0 || num_blocks <= 0) return ATTN_ERR_INVALID_ARG;
  if (max_blocks > kMaxPoolBlocks || num_blocks > kMaxPoolBlocks) return ATTN_ERR_UNSUPPORTED;
  if (block_size != decode::kBlock) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

int decode_fp8_entry(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                     const int32_t* seq_lens, int B, int Hq, int Hkv, int d, int block_size, int max_blocks,
                     int num_blocks, int num_splits, float k_scale, float v_scale, void* o, cudaStream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || block_size <= 0) return ATTN_ERR_INVALID_ARG;
  if (!(k_scale > 0.f) || !std::isfinite(k_scale) || !(v_scale > 0.f) || !std::isfinite(v_scale))
    return ATTN_ERR_INVALID_ARG;
  int rc = check_paged_common(B, Hq, Hkv, d, block_size, max_blocks, num_blocks);
  if (rc != ATTN_OK || B == 0) return rc;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || block_table == nullptr || seq_lens == nullptr ||
      o == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (d != decode::kFp8D) return ATTN_ERR_UNSUPPORTED;
  if (Hq / Hkv > 8) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  rc = current_device_state(&st);
  if (rc != ATTN_OK) return rc;
  return launch_decode_fp8(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, max_blocks, num_blocks,
                           num_splits, k_scale, v_scale, o, stream, st);
}

// o_part / lse_part non-null: the partial form (o is then unused and may be null).
int decode_entry(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                 const int32_t* seq_lens, int B, int Hq, int Hkv, int d, int block_size, int max_blocks,
                 int num_blocks, int num_splits, void* o, cudaStream_t stream, float* o_part = nullptr,
                 float* lse_part = nullptr) {
  int rc = check_paged_common(B, Hq, Hkv, d, block_size, max_blocks, num_blocks);
  if (rc != ATTN_OK || B == 0) return rc;
  const bool partial = o_part != nullptr || lse_part != nullptr;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || block_table == nullptr || seq_lens == nullptr ||
      (partial ? (o_part == nullptr || lse_part == nullptr) : o == nullptr))
    return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Hq / Hkv > 8) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return ATTN_ERR_UNSUPPORTED;
  if (partial ? (!aligned16(o_part) || (reinterpret_cast<uintptr_t>(lse_part) & 3u)) : !aligned16(o))
    return ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  rc = current_device_state(&st);
  if (rc != ATTN_OK) return rc;
  if (d == 64)
    return launch_decode<64>(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, max_blocks, num_blocks,
                             num_splits, o, stream, st, o_part, lse_part);
  return launch_decode<128>(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, max_blocks, num_blocks,
                            num_splits, o, stream, st, o_part, lse_part);
}

// Merge R partials per (sequence, query head) row into bf16 O with the
// decode's LSE combine kernel (every partial of a row taken).
int lse_merge_entry(const float* o_parts, const float* lse_parts, int R, int B, int Hq, int d, void* o,
                    cudaStream_t stream) {
  if (R <= 0 || B < 0 || Hq <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (B == 0) return ATTN_OK;
  if (o_parts == nullptr || lse_parts == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (R > 65535 || static_cast<long long>(B) * Hq > (1LL << 30)) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(o_parts) || !aligned16(o) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u))
    return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  int rc = current_device_state(&st);
  if (rc != ATTN_OK) return rc;
  decode::Params p;
  p.q = nullptr;
  p.block_table = nullptr;
  p.seq_lens = nullptr;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.part_o = const_cast<float*>(o_parts);
  p.part_lse = const_cast<float*>(lse_parts);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hq;
  p.max_blocks = 1;
  p.num_blocks = 1;
  p.num_splits = R;
  p.chunk = 1;
  p.scale_log2 = 1.0f;
  if (d == 64) return launch_combine<64>(p, nullptr, o, nullptr, stream);
  return launch_combine<128>(p, nullptr, o, nullptr, stream);
}

int prefill_paged_entry(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                        const int32_t* seq_lens, const int32_t* cu_seqlens_q, int B, int Hq, int Hkv, int d,
                        int block_size, int max_blocks, int num_blocks, int max_seqlen_q, int total_q, int causal,
                        float scale, void* o, float* lse, cudaStream_t stream) {
  if (max_seqlen_q < 0 || total_q < 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  int rc = check_paged_common(B, Hq, Hkv, d, block_size, max_blocks, num_blocks);
  if (rc != ATTN_OK) return rc;
  if (B == 0 || total_q == 0 || max_seqlen_q == 0) return ATTN_OK;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || block_table == nullptr || seq_lens == nullptr ||
      cu_seqlens_q == nullptr || o == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return ATTN_ERR_UNSUPPORTED;
  if ((lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u))
    return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  rc = current_device_state(&st);
  if (rc != ATTN_OK) return rc;
  if (d == 64)
    return launch_prefill_paged<64>(q, k_cache, v_cache, block_table, seq_lens, cu_seqlens_q, o, lse, B,
                                    max_seqlen_q, total_q, Hq, Hkv, max_blocks, num_blocks, causal, scale, stream);
  return launch_prefill_paged<128>(q, k_cache, v_cache, block_table, seq_lens, cu_seqlens_q, o, lse, B,
                                   max_seqlen_q, total_q, Hq, Hkv, max_blocks, num_blocks, causal, scale, stream);
}

}  // namespace
}  // namespace attn

extern "C" int paged_attn_decode_fp8(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_table, const int32_t* seq_lens, int B, int Hq, int Hkv,
                                     int d, int block_size, int max_blocks, int num_splits, float k_scale,
                                     float v_scale, void* o, attn_stream_t stream) {
  return decode_fp8_entry(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size, max_blocks,
                          kMaxPoolBlocks, num_splits, k_scale, v_scale, o, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int paged_attn_decode_fp8_checked(const void* q, const void* k_cache, const void* v_cache,
                                             const int32_t* block_table, const int32_t* seq_lens, int B, int Hq,
                                             int Hkv, int d, int block_size, int max_blocks, int num_blocks,
                                             int num_splits, float k_scale, float v_scale, void* o,
                                             attn_stream_t stream) {
  return decode_fp8_entry(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size, max_blocks,
                          num_blocks, num_splits, k_scale, v_scale, o, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                        int T, int S, int d, int causal, float scale, attn_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (B < 0 || T < 0 || S < 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return ATTN_OK;
  if (q == nullptr || o == nullptr || (S > 0 && (k == nullptr || v == nullptr))) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(o) || (S > 0 && (!aligned16(k) || !aligned16(v)))) return ATTN_ERR_UNSUPPORTED;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  int rc = current_device_state(&st);
  if (rc != ATTN_OK) return rc;
  if (S == 0) {  // no key at all: O = 0, LSE = -inf
    const size_t n_o = static_cast<size_t>(B) * T * Hq * d;
    const size_t n_lse = static_cast<size_t>(B) * Hq * T;
    fill_no_keys<<<st->sms * 4, 256, 0, stream>>>(static_cast<__nv_bfloat16*>(o), lse, n_o, n_lse);
    return launch_status();
  }
  if (d == 64) return launch_prefill<64>(q, k, v, o, lse, B, Hq, Hkv, T, S, causal, scale, stream);
  return launch_prefill<128>(q, k, v, o, lse, B, Hq, Hkv, T, S, causal, scale, stream);
}

extern "C" int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                               const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B, int max_seqlen_q,
                               int total_q, int total_k, int Hq, int Hkv, int d, int causal, float scale,
                               attn_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (B < 0 || max_seqlen_q < 0 || total_q < 0 || total_k < 0 || Hq <= 0 || Hkv <= 0 || d <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || total_q == 0 || max_seqlen_q == 0) return ATTN_OK;
  if (q == nullptr || o == nullptr || cu_seqlens_q == nullptr || cu_seqlens_k == nullptr) return ATTN_ERR_INVALID_ARG;
  if (total_k > 0 && (k == nullptr || v == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(o) || (total_k > 0 && (!aligned16(k) || !aligned16(v)))) return ATTN_ERR_UNSUPPORTED;
  if ((lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  int rc = current_device_state(&st);
  if (rc != ATTN_OK) return rc;
  if (total_k == 0) {  // no key anywhere: O = 0, LSE = -inf
    const size_t n_o = static_cast<size_t>(total_q) * Hq * d;
    const size_t n_lse = static_cast<size_t>(Hq) * total_q;
    fill_no_keys<<<st->sms * 4, 256, 0, stream>>>(static_cast<__nv_bfloat16*>(o), lse, n_o, n_lse);
    return launch_status();
  }
  if (d == 64)
    return launch_prefill_varlen<64>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, total_q, total_k,
                                     Hq, Hkv, causal, scale, stream);
  return launch_prefill_varlen<128>(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, total_q, total_k,
                                    Hq, Hkv, causal, scale, stream);
}

extern "C" int paged_attn_prefill(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* block_table, const int32_t* seq_lens, const int32_t* cu_seqlens_q,
                                  int B, int Hq, int Hkv, int d, int block_size, int max_blocks, int max_seqlen_q,
                                  int total_q, int causal, float scale, void* o, float* lse, attn_stream_t stream) {
  return prefill_paged_entry(q, k_cache, v_cache, block_table, seq_lens, cu_seqlens_q, B, Hq, Hkv, d, block_size,
                             max_blocks, kMaxPoolBlocks, max_seqlen_q, total_q, causal, scale, o, lse,
                             reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int paged_attn_prefill_checked(const void* q, const void* k_cache, const void* v_cache,
                                          const int32_t* block_table, const int32_t* seq_lens,
                                          const int32_t* cu_seqlens_q, int B, int Hq, int Hkv, int d, int block_size,
                                          int max_blocks, int num_blocks, int max_seqlen_q, int total_q, int causal,
                                          float scale, void* o, float* lse, attn_stream_t stream) {
  return prefill_paged_entry(q, k_cache, v_cache, block_table, seq_lens, cu_seqlens_q, B, Hq, Hkv, d, block_size,
                             max_blocks, num_blocks, max_seqlen_q, total_q, causal, scale, o, lse,
                             reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int paged_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* block_table, const int32_t* seq_lens, int B, int Hq, int Hkv, int d,
                                 int block_size, int max_blocks, int num_splits, void* o, attn_stream_t stream) {
  return decode_entry(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size, max_blocks,
                      kMaxPoolBlocks, num_splits, o, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int paged_attn_decode_checked(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_table, const int32_t* seq_lens, int B, int Hq, int Hkv,
                                         int d, int block_size, int max_blocks, int num_blocks, int num_splits,
                                         void* o, attn_stream_t stream) {
  return decode_entry(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size, max_blocks,
                      num_blocks, num_splits, o, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int paged_attn_decode_partial(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_table, const int32_t* seq_lens, int B, int Hq, int Hkv,
                                         int d, int block_size, int max_blocks, int num_blocks, int num_splits,
                                         float* o_part, float* lse_part, attn_stream_t stream) {
  if (o_part == nullptr || lse_part == nullptr) return ATTN_ERR_INVALID_ARG;
  return decode_entry(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size, max_blocks,
                      num_blocks, num_splits, nullptr, reinterpret_cast<cudaStream_t>(stream), o_part, lse_part);
}

extern "C" int attn_lse_merge(const float* o_parts, const float* lse_parts, int R, int B, int Hq, int d, void* o,
                              attn_stream_t stream) {
  return lse_merge_entry(o_parts, lse_parts, R, B, Hq, d, o, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int attn_check_support(int device) {
  DeviceState* st = nullptr;
  return probe_device(device, &st);
}

extern "C" const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK:
      return "ok";
    case ATTN_ERR_INVALID_ARG:
      return "invalid argument";
    case ATTN_ERR_UNSUPPORTED:
      return "unsupported (shape, alignment or device)";
    case ATTN_ERR_CUDA:
      return "CUDA error";
    case ATTN_ERR_TIMEOUT:
      return "device-side wait timed out";
    default:
      return "unknown status";
  }
}

namespace attn {
namespace {
// One thread waits on a barrier that expects one arrival that never comes.
__global__ void selftest_bounded_wait_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag);  // gives up after the limit
}
}  // namespace
}  // namespace attn

extern "C" int attn_selftest_bounded_wait(attn_stream_t stream_) {
  attn::selftest_bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream_)>>>();
  return attn::launch_status();
}

extern "C" int attn_read_device_status(int* out, int clear) {
  if (out == nullptr) return ATTN_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, attn::g_devstatus, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  *out = v;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(attn::g_devstatus, &zero, sizeof(int)) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
  }
  return ATTN_OK;
}

// ---------------------------------------------------------------------------
// paged_attn_decode_noalloc: the same kernels with their split partials in a
// fixed scratch array compiled into the library instead of pool memory.
// ---------------------------------------------------------------------------
namespace attn {
namespace {

// Scratch for the split partials of paged_attn_decode_noalloc.  In host code
// this name is only a stand-in for the device array; its device address is
// looked up with cudaGetSymbolAddress once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

struct NoAllocState {
  bool ready = false;
  void* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};
NoAllocState g_noalloc[kMaxDevices];

// Once per device, with that device current: shared-memory limits of the
// decode kernels and the scratch array's device address.  No allocation.
int prepare_noalloc(int dev, void** scratch) {
  std::lock_guard<std::mutex> lock(g_mu);
  NoAllocState& na = g_noalloc[dev];
  if (!na.ready) {
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(decode::paged_decode_split<64>),
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(decode::smem_bytes<64>())) != cudaSuccess ||
        cudaFuncSetAttribute(reinterpret_cast<const void*>(decode::paged_decode_split<128>),
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(decode::smem_bytes<128>())) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    na.scratch = ptr;
    na.ready = true;
  }
  *scratch = na.scratch;
  return ATTN_OK;
}

template <int D>
int launch_decode_noalloc(const void* q, const void* kc, const void* vc, const int32_t* table,
                          const int32_t* lens, int B, int Hq, int Hkv, int max_blocks, int num_splits, void* o,
                          cudaStream_t stream, int sms, void* scratch) {
  const int groups = (Hkv + decode::kKH - 1) / decode::kKH;
  const size_t row_bytes = static_cast<size_t>(B) * Hq * (D + 1) * sizeof(float);  // partials of one split
  if (num_splits <= 0) {
    // the automatic choice, lowered to what the scratch holds (1 split needs none)
    num_splits = auto_splits(B, groups, max_blocks, sms);
    const size_t fit = ATTN_NOALLOC_SCRATCH_BYTES / row_bytes;
    if (static_cast<size_t>(num_splits) > fit) num_splits = fit >= 2 ? static_cast<int>(fit) : 1;
  }
  if (num_splits > max_blocks) num_splits = max_blocks;
  const int chunk = (max_blocks + num_splits - 1) / num_splits;
  num_splits = (max_blocks + chunk - 1) / chunk;
  if (num_splits > 65535 || groups > 65535 || B > 65535) return ATTN_ERR_UNSUPPORTED;
  const size_t rows = static_cast<size_t>(num_splits) * B * Hq;
  if (num_splits > 1 && num_splits * row_bytes > ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_UNSUPPORTED;
  CUtensorMap mk, mv;
  if (make_map_decode_bf16(&mk, kc, Hkv, D, kMaxPoolBlocks) || make_map_decode_bf16(&mv, vc, Hkv, D, kMaxPoolBlocks))
    return ATTN_ERR_CUDA;

  decode::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.block_table = table;
  p.seq_lens = lens;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.part_o = num_splits > 1 ? static_cast<float*>(scratch) : nullptr;
  p.part_lse = num_splits > 1 ? static_cast<float*>(scratch) + rows * D : nullptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.max_blocks = max_blocks;
  p.num_blocks = kMaxPoolBlocks;
  p.num_splits = num_splits;
  p.chunk = chunk;
  p.scale_log2 = (1.0f / std::sqrt(static_cast<float>(D))) * 1.4426950408889634f;

  dim3 grid(num_splits, groups, B);
  decode::paged_decode_split<D><<<grid, (decode::kKH + 1) * 32, decode::smem_bytes<D>(), stream>>>(mk, mv, p);
  int rc = launch_status();
  if (rc == ATTN_OK && num_splits > 1) rc = launch_combine<D>(p, lens, o, nullptr, stream);
  return rc;
}

}  // namespace
}  // namespace attn

extern "C" int paged_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_table, const int32_t* seq_lens, int B, int Hq,
                                         int Hkv, int d, int block_size, int max_blocks, int num_splits, void* o,
                                         attn_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (B < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || block_size <= 0) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (B == 0) return ATTN_OK;
  if (max_blocks <= 0) return ATTN_ERR_INVALID_ARG;
  if (max_blocks > kMaxPoolBlocks) return ATTN_ERR_UNSUPPORTED;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || block_table == nullptr || seq_lens == nullptr ||
      o == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (block_size != decode::kBlock) return ATTN_ERR_UNSUPPORTED;
  if (Hq / Hkv > 8) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o)) return ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  DeviceState* st = nullptr;
  int rc = probe_device(dev, &st);
  if (rc != ATTN_OK) return rc;
  void* scratch = nullptr;
  rc = prepare_noalloc(dev, &scratch);
  if (rc != ATTN_OK) return rc;
  if (d == 64)
    return launch_decode_noalloc<64>(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, max_blocks,
                                     num_splits, o, stream, st->sms, scratch);
  return launch_decode_noalloc<128>(q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, max_blocks,
                                    num_splits, o, stream, st->sms, scratch);
}

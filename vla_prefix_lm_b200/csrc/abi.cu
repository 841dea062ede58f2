// abi.cu -- the extern "C" entry points of libpiattn.so (declared in
// include/pi_attn.h): argument validation, TMA tensor-map encoding, dispatch
// to the kernels, and the device status word.
//
// Validation happens entirely on the host, before anything is enqueued: an
// entry point that returns an error has launched nothing.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "../../include/pi_attn.h"
#include "launch.h"
#include "mask.cuh"

namespace {

using namespace piattn;

constexpr unsigned long long kDefaultWaitLimit = 1ull << 31;

// The bound on every device-side wait, in SM cycles: PIATTN_WATCHDOG_CYCLES
// when set (a positive integer) at load time, else 2^31 (about a second).
unsigned long long initial_wait_limit() {
  const char* e = std::getenv("PIATTN_WATCHDOG_CYCLES");
  if (e && *e) {
    char* end = nullptr;
    const unsigned long long v = std::strtoull(e, &end, 10);
    if (end && *end == '\0' && v > 0) return v;
  }
  return kDefaultWaitLimit;
}
std::atomic<unsigned long long> g_wait_limit{initial_wait_limit()};

// An NVTX range around each entry point that enqueues work (free unless a
// profiler is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// The device status word (one per device context).  Its address is looked up
// on every call (a host-side table lookup), so it stays right after the
// context is reset and the module reloaded.
__device__ int g_status;

int* status_ptr() {
  void* p = nullptr;
  return cudaGetSymbolAddress(&p, g_status) == cudaSuccess ? static_cast<int*>(p) : nullptr;
}

bool make_ctl(DevCtl* ctl) {
  ctl->status = status_ptr();
  ctl->wait_limit = g_wait_limit.load();
  return ctl->status != nullptr;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// A [batch][rows][256] bf16 tensor viewed as 4-D (64, rows, 4, batch): the
// row stride is 512 B and dimension 2 walks the four 64-column blocks of a
// row (stride 128 B), so one box (64, box_rows, 4, 1) lands in shared memory
// as 4 blocks of [box_rows x 64] with the 128-byte swizzle -- the operand
// layout of the tensor-core kernels.  A box of 2 blocks brings half the
// columns (the CTA-pair kernel's V quarters).  Rows past `rows` read as zero and are
// clipped on stores.
bool encode_rows(CUtensorMap* map, const void* base, uint64_t rows, uint64_t batch,
                 uint32_t box_rows, uint32_t box_blocks = 4) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, rows, 4, batch};
  cuuint64_t strides[3] = {256 * 2, 64 * 2, 256 * 2 * rows};
  cuuint32_t box[4] = {64, box_rows, box_blocks, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A [batch][rows][blocks * 64] bf16 tensor (row pitch `pitch` bytes) viewed as
// 4-D (64, rows, blocks, batch), box (64, box_rows, box_blocks, 1), 128-byte
// swizzle: the general form of encode_rows for the backward's workspace.
bool encode_view(CUtensorMap* map, const void* base, uint64_t rows, uint64_t blocks,
                 uint64_t batch, uint64_t pitch, uint32_t box_rows, uint32_t box_blocks) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, rows, blocks, batch};
  cuuint64_t strides[3] = {pitch, 64 * 2, pitch * rows};
  cuuint32_t box[4] = {64, box_rows, box_blocks, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A [batch][rows][cols] bf16 tensor (row pitch `pitch` bytes) viewed as 3-D
// (cols, rows, batch), box (32, 32, 1) with the 64-byte swizzle: 32-row by
// 32-column boxes whose 64-byte rows carry their 16-byte chunks at
// chunk ^ ((row / 2) % 4); rows past `rows` of a batch element are clipped.
bool encode_rows64b(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                    uint64_t batch, uint64_t pitch) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, batch};
  cuuint64_t strides[2] = {pitch, pitch * rows};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The backward runs on tensor cores for the forward's tensor-core geometry
// (bf16, one KV head, head_dim 256); every other shape uses the SIMT kernels.
bool backward_on_tensor_cores(const pi_attn_desc* d) {
  return d->dtype == PI_BF16 && d->Hkv == 1 && d->d == 256 &&
         (d->Hq == 1 || d->Hq == 2 || d->Hq == 4 || d->Hq == 8 || d->Hq == 16);
}

int check_desc(const pi_attn_desc* d, bool suffix) {
  if (!d) return PI_ERR_ARG;
  if (d->B < 0 || d->Sq < 0 || d->P < 0 || d->Hq <= 0 || d->Hkv <= 0 || d->d <= 0)
    return PI_ERR_ARG;
  if (!suffix && d->P != 0) return PI_ERR_ARG;
  if (d->Hq % d->Hkv != 0) return PI_ERR_ARG;
  if (!std::isfinite(d->softmax_scale) || !(d->softmax_scale > 0.f)) return PI_ERR_ARG;
  if (d->mask_batch_stride < 0 || (d->mask_batch_stride != 0 && d->mask_batch_stride < d->Sq))
    return PI_ERR_ARG;
  if (d->Sq > kMaxTokens) return PI_ERR_UNSUPPORTED;
  if (d->dtype == PI_BF16) {
    if (d->Hkv != 1 || d->d != 256) return PI_ERR_UNSUPPORTED;
    if (!(d->Hq == 1 || d->Hq == 2 || d->Hq == 4 || d->Hq == 8 || d->Hq == 16))
      return PI_ERR_UNSUPPORTED;
    if ((long long)d->P * d->Hq >= (1ll << 31)) return PI_ERR_UNSUPPORTED;
  } else if (d->dtype == PI_F32) {
    if (!(d->d == 32 || d->d == 64 || d->d == 128 || d->d == 256)) return PI_ERR_UNSUPPORTED;
  } else {
    return PI_ERR_UNSUPPORTED;
  }
  return PI_OK;
}

int launched(cudaError_t e) { return e == cudaSuccess ? PI_OK : PI_ERR_CUDA; }

int check_backward_desc(const pi_attn_desc* d) {
  if (!d) return PI_ERR_ARG;
  if (d->B < 0 || d->Sq < 0 || d->P != 0 || d->Hq <= 0 || d->Hkv <= 0 || d->d <= 0)
    return PI_ERR_ARG;
  if (d->Hq % d->Hkv != 0) return PI_ERR_ARG;
  if (!std::isfinite(d->softmax_scale) || !(d->softmax_scale > 0.f)) return PI_ERR_ARG;
  if (d->mask_batch_stride < 0 || (d->mask_batch_stride != 0 && d->mask_batch_stride < d->Sq))
    return PI_ERR_ARG;
  if (d->dtype != PI_BF16 && d->dtype != PI_F32) return PI_ERR_UNSUPPORTED;
  if (d->Sq > kMaxTokens || d->d % 32 != 0 || d->d > 256) return PI_ERR_UNSUPPORTED;
  if ((long long)d->B * d->Sq * d->Hq / 8 >= (1ll << 31)) return PI_ERR_UNSUPPORTED;
  return PI_OK;
}

}  // namespace

extern "C" {

namespace {
bool tail_split_applies(const pi_attn_desc* d) {
  return d->dtype == PI_BF16 && d->mask_batch_stride == 0;
}

int prefill_impl(const pi_attn_desc* d, const void* q, const void* k, const void* v,
                 const uint8_t* ar_mask, const int32_t* segment_ids, void* out, float* lse,
                 void* workspace, size_t ws_bytes, pi_stream_t stream) {
  int rc = check_desc(d, false);
  if (rc != PI_OK) return rc;
  if (workspace != nullptr && tail_split_applies(d)) {
    if (!aligned16(workspace)) return PI_ERR_ALIGN;
    if (ws_bytes < tc_prefill_tail_bytes()) return PI_ERR_ARG;
  }
  if (d->B == 0 || d->Sq == 0) return PI_OK;
  if (!q || !k || !v || !ar_mask || !out) return PI_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return PI_ERR_ALIGN;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return PI_ERR_ALIGN;
  if (segment_ids && (reinterpret_cast<uintptr_t>(segment_ids) & 3u)) return PI_ERR_ALIGN;
  DevCtl ctl;
  if (!make_ctl(&ctl)) return PI_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->dtype == PI_F32) {
    SimtParams p{};
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.ar = ar_mask;
    p.seg = segment_ids;
    p.mask_bs = d->mask_batch_stride;
    p.out = static_cast<float*>(out);
    p.lse = lse;
    p.B = d->B; p.Sq = d->Sq; p.P = 0; p.Hq = d->Hq; p.Hkv = d->Hkv; p.d = d->d;
    p.scale = d->softmax_scale;
    return launched(launch_simt_f32(p, ctl, st));
  }
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  const uint64_t rows = (uint64_t)d->Sq * d->Hq;
  if (!encode_rows(&p.map_q, q, rows, d->B, 128) ||
      !encode_rows(&p.map_k, k, d->Sq, d->B, 64) ||
      !encode_rows(&p.map_vh, v, d->Sq, d->B, 64, 2) ||
      !encode_rows(&p.map_o, out, rows, d->B, 32, 1))
    return PI_ERR_CUDA;
  p.map_kc = p.map_k;
  p.map_vch = p.map_vh;
  p.ar = ar_mask;
  p.seg = segment_ids;
  p.mask_bs = d->mask_batch_stride;
  p.lse = lse;
  p.ws = tail_split_applies(d) ? static_cast<float*>(workspace) : nullptr;
  p.out_ptr = out;
  p.B = d->B; p.Sq = d->Sq; p.P = 0; p.Hq = d->Hq;
  p.n_splits = 1;
  p.scale = d->softmax_scale;
  p.scale_log2 = d->softmax_scale * 1.4426950408889634f;
  return launched(launch_tc_pair(p, false, ctl, st));
}
}  // namespace

int pi_attn_prefill(const pi_attn_desc* d, const void* q, const void* k, const void* v,
                    const uint8_t* ar_mask, const int32_t* segment_ids, void* out, float* lse,
                    pi_stream_t stream) {
  NvtxRange range("pi_attn_prefill");
  return prefill_impl(d, q, k, v, ar_mask, segment_ids, out, lse, nullptr, 0, stream);
}

size_t pi_attn_prefill_workspace_bytes(const pi_attn_desc* d) {
  if (check_desc(d, false) != PI_OK || !tail_split_applies(d)) return 0;
  return tc_prefill_tail_bytes();
}

int pi_attn_prefill_tail_splits(const pi_attn_desc* d) {
  if (check_desc(d, false) != PI_OK || !tail_split_applies(d) || d->B == 0 || d->Sq == 0)
    return 1;
  return tc_prefill_tail_splits(d->B, d->Sq, d->Hq);
}

int pi_attn_prefill_ws(const pi_attn_desc* d, const void* q, const void* k, const void* v,
                       const uint8_t* ar_mask, const int32_t* segment_ids, void* out, float* lse,
                       void* workspace, size_t ws_bytes, pi_stream_t stream) {
  NvtxRange range("pi_attn_prefill_ws");
  return prefill_impl(d, q, k, v, ar_mask, segment_ids, out, lse, workspace, ws_bytes, stream);
}

size_t pi_attn_suffix_workspace_bytes(const pi_attn_desc* d) {
  if (check_desc(d, true) != PI_OK) return 0;
  if (d->dtype != PI_BF16 || d->B == 0 || d->Sq == 0) return 0;
  if (decode_applies(d->Sq, d->Hq)) return 0;
  return tc_suffix_workspace_bytes(d->B, d->Sq, d->P, d->Hq);
}

int pi_attn_suffix_masked(const pi_attn_desc* d, const void* q_suf, const void* k_suf,
                          const void* v_suf, const void* k_cache, const void* v_cache,
                          const uint8_t* ar_mask_suf, const int32_t* segment_ids_suf,
                          const uint8_t* cache_valid, void* out, void* workspace,
                          size_t ws_bytes, pi_stream_t stream) {
  NvtxRange range("pi_attn_suffix_masked");
  int rc = check_desc(d, true);
  if (rc != PI_OK) return rc;
  if (d->B == 0 || d->Sq == 0) return PI_OK;
  if (!q_suf || !k_suf || !v_suf || !ar_mask_suf || !out) return PI_ERR_ARG;
  if (d->P > 0 && (!k_cache || !v_cache)) return PI_ERR_ARG;
  if (!aligned16(q_suf) || !aligned16(k_suf) || !aligned16(v_suf) || !aligned16(out) ||
      (d->P > 0 && (!aligned16(k_cache) || !aligned16(v_cache))))
    return PI_ERR_ALIGN;
  if (segment_ids_suf && (reinterpret_cast<uintptr_t>(segment_ids_suf) & 3u)) return PI_ERR_ALIGN;
  if (d->P == 0) cache_valid = nullptr;
  DevCtl ctl;
  if (!make_ctl(&ctl)) return PI_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->dtype == PI_F32) {
    SimtParams p{};
    p.q = static_cast<const float*>(q_suf);
    p.k = static_cast<const float*>(k_suf);
    p.v = static_cast<const float*>(v_suf);
    p.kc = static_cast<const float*>(k_cache);
    p.vc = static_cast<const float*>(v_cache);
    p.ar = ar_mask_suf;
    p.seg = segment_ids_suf;
    p.mask_bs = d->mask_batch_stride;
    p.out = static_cast<float*>(out);
    p.lse = nullptr;
    p.cache_valid = cache_valid;
    p.B = d->B; p.Sq = d->Sq; p.P = d->P; p.Hq = d->Hq; p.Hkv = d->Hkv; p.d = d->d;
    p.scale = d->softmax_scale;
    return launched(launch_simt_f32(p, ctl, st));
  }
  if (decode_applies(d->Sq, d->Hq)) {
    // Few query rows: the cache is spread over a cluster of CTAs per batch
    // element and merged on chip (no workspace).
    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    if (!encode_rows(&p.map_k, k_suf, d->Sq, d->B, kDecodeTileKeys) ||
        !encode_rows(&p.map_v, v_suf, d->Sq, d->B, kDecodeTileKeys))
      return PI_ERR_CUDA;
    if (d->P > 0) {
      if (!encode_rows(&p.map_kc, k_cache, d->P, d->B, kDecodeTileKeys) ||
          !encode_rows(&p.map_vc, v_cache, d->P, d->B, kDecodeTileKeys))
        return PI_ERR_CUDA;
    } else {
      p.map_kc = p.map_k;
      p.map_vc = p.map_v;
    }
    p.q = static_cast<const __nv_bfloat16*>(q_suf);
    p.ar = ar_mask_suf;
    p.seg = segment_ids_suf;
    p.mask_bs = d->mask_batch_stride;
    p.cache_valid = cache_valid;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.B = d->B; p.Sq = d->Sq; p.P = d->P; p.Hq = d->Hq;
    p.scale_log2 = d->softmax_scale * 1.4426950408889634f;
    return launched(launch_decode(p, ctl, st));
  }
  const int splits = tc_suffix_splits(d->B, d->Sq, d->P, d->Hq);
  const size_t need = tc_suffix_workspace_bytes(d->B, d->Sq, d->P, d->Hq);
  if (need > 0) {
    if (!workspace || ws_bytes < need) return PI_ERR_ARG;
    if (!aligned16(workspace)) return PI_ERR_ALIGN;
  }
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  const uint64_t rows = (uint64_t)d->Sq * d->Hq;
  if (!encode_rows(&p.map_q, q_suf, rows, d->B, 128) ||
      !encode_rows(&p.map_k, k_suf, d->Sq, d->B, 64) ||
      !encode_rows(&p.map_vh, v_suf, d->Sq, d->B, 64, 2) ||
      !encode_rows(&p.map_o, out, rows, d->B, 32, 1))
    return PI_ERR_CUDA;
  if (d->P > 0) {
    if (!encode_rows(&p.map_kc, k_cache, d->P, d->B, 64) ||
        !encode_rows(&p.map_vch, v_cache, d->P, d->B, 64, 2))
      return PI_ERR_CUDA;
  } else {
    p.map_kc = p.map_k;
    p.map_vch = p.map_vh;
  }
  p.ar = ar_mask_suf;
  p.seg = segment_ids_suf;
  p.mask_bs = d->mask_batch_stride;
  p.lse = nullptr;
  p.cache_valid = cache_valid;
  p.ws = static_cast<float*>(workspace);
  p.out_ptr = out;
  p.B = d->B; p.Sq = d->Sq; p.P = d->P; p.Hq = d->Hq;
  p.n_splits = splits;
  p.scale = d->softmax_scale;
  p.scale_log2 = d->softmax_scale * 1.4426950408889634f;
  return launched(launch_tc_pair(p, true, ctl, st));
}

int pi_attn_suffix(const pi_attn_desc* d, const void* q_suf, const void* k_suf,
                   const void* v_suf, const void* k_cache, const void* v_cache,
                   const uint8_t* ar_mask_suf, void* out, void* workspace, size_t ws_bytes,
                   pi_stream_t stream) {
  NvtxRange range("pi_attn_suffix");
  return pi_attn_suffix_masked(d, q_suf, k_suf, v_suf, k_cache, v_cache, ar_mask_suf, nullptr,
                               nullptr, out, workspace, ws_bytes, stream);
}

int pi_rope_inplace(const pi_rope_desc* d, void* q, void* k, const uint8_t* token_mask,
                    const uint8_t* prefix_mask, int32_t* positions_out, pi_stream_t stream) {
  NvtxRange range("pi_rope_inplace");
  if (!d) return PI_ERR_ARG;
  if (d->B < 0 || d->S < 0 || d->P < 0 || d->Hq <= 0 || d->Hkv <= 0 || d->d <= 0)
    return PI_ERR_ARG;
  if (!(d->base > 1.f) || !std::isfinite(d->base)) return PI_ERR_ARG;
  if (d->dtype != PI_BF16 && d->dtype != PI_F32) return PI_ERR_UNSUPPORTED;
  if (d->d > 256 || d->d % 16 != 0 || d->B > 65535) return PI_ERR_UNSUPPORTED;
  if (((size_t)d->Hq + (k ? (size_t)d->Hkv : 0)) * d->d * (d->dtype == PI_F32 ? 4 : 2) >
      rope_max_smem())
    return PI_ERR_UNSUPPORTED;
  if (d->mask_batch_stride < 0 || (d->mask_batch_stride != 0 && d->mask_batch_stride < d->S))
    return PI_ERR_ARG;
  if (d->prefix_batch_stride < 0 ||
      (d->prefix_batch_stride != 0 && d->prefix_batch_stride < d->P))
    return PI_ERR_ARG;
  if (d->B == 0 || d->S == 0) return PI_OK;
  if (!q || !token_mask) return PI_ERR_ARG;
  if (d->P > 0 && !prefix_mask) return PI_ERR_ARG;
  if (!aligned16(q) || (k && !aligned16(k))) return PI_ERR_ALIGN;
  if (positions_out && (reinterpret_cast<uintptr_t>(positions_out) & 3u)) return PI_ERR_ALIGN;
  RopeParams p;
  p.q = q;
  p.k = k;
  p.tmask = token_mask;
  p.tmask_bs = d->mask_batch_stride;
  p.pmask = d->P > 0 ? prefix_mask : nullptr;
  p.pmask_bs = d->prefix_batch_stride;
  p.pos_out = positions_out;
  p.B = d->B; p.S = d->S; p.P = d->P; p.Hq = d->Hq; p.Hkv = d->Hkv; p.d = d->d;
  p.base = d->base;
  p.f32 = d->dtype == PI_F32;
  DevCtl ctl;
  if (!make_ctl(&ctl)) return PI_ERR_CUDA;
  return launched(launch_rope(p, ctl, static_cast<cudaStream_t>(stream)));
}

int pi_euler_update(float* x, const void* v, int32_t v_dtype, float dt, int64_t n,
                    pi_stream_t stream) {
  NvtxRange range("pi_euler_update");
  if (n < 0 || !std::isfinite(dt)) return PI_ERR_ARG;
  if (v_dtype != PI_BF16 && v_dtype != PI_F32) return PI_ERR_UNSUPPORTED;
  if (n == 0) return PI_OK;
  if (!x || !v) return PI_ERR_ARG;
  if (!aligned16(x) || !aligned16(v)) return PI_ERR_ALIGN;
  return launched(launch_euler(x, v, v_dtype == PI_F32, dt, n, static_cast<cudaStream_t>(stream)));
}

size_t pi_attn_prefill_backward_workspace_bytes(const pi_attn_desc* d) {
  if (check_backward_desc(d) != PI_OK || d->B == 0 || d->Sq == 0) return 0;
  if (backward_on_tensor_cores(d)) return bwd_tc_plan(d->B, d->Sq, d->Hq, sm_count()).bytes;
  return bwd_workspace_bytes(d->B, d->Sq, d->Hq);
}

int pi_attn_prefill_backward(const pi_attn_desc* d, const void* q, const void* k, const void* v,
                             const uint8_t* ar_mask, const int32_t* segment_ids, const void* out,
                             const float* lse, const void* dout, float* dq, float* dk, float* dv,
                             void* workspace, size_t ws_bytes, pi_stream_t stream) {
  NvtxRange range("pi_attn_prefill_backward");
  const int rc = check_backward_desc(d);
  if (rc != PI_OK) return rc;
  if (d->B == 0 || d->Sq == 0) return PI_OK;
  if (!q || !k || !v || !ar_mask || !out || !lse || !dout || !dq || !dk || !dv || !workspace)
    return PI_ERR_ARG;
  const bool tc = backward_on_tensor_cores(d);
  const BwdTcPlan plan = tc ? bwd_tc_plan(d->B, d->Sq, d->Hq, sm_count()) : BwdTcPlan{};
  const size_t need = tc ? plan.bytes : bwd_workspace_bytes(d->B, d->Sq, d->Hq);
  if (ws_bytes < need) return PI_ERR_ARG;
  for (const void* ptr : {q, k, v, out, dout, (const void*)dq, (const void*)dk, (const void*)dv,
                          (const void*)workspace})
    if (!aligned16(ptr)) return PI_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (segment_ids && (reinterpret_cast<uintptr_t>(segment_ids) & 3u)))
    return PI_ERR_ALIGN;
  if (tc) {
    DevCtl ctl;
    if (!make_ctl(&ctl)) return PI_ERR_CUDA;
    BwdTcParams t;
    std::memset(&t, 0, sizeof(t));
    uint8_t* w = static_cast<uint8_t*>(workspace);
    const uint64_t rows = (uint64_t)d->Sq * d->Hq;
    const uint64_t pitch = (uint64_t)plan.Skp * 2;
    t.D = reinterpret_cast<float*>(w + plan.off_D);
    t.P = reinterpret_cast<__nv_bfloat16*>(w + plan.off_P);
    t.dS = reinterpret_cast<__nv_bfloat16*>(w + plan.off_dS);
    t.part = plan.n_chunks > 1 ? reinterpret_cast<float*>(w + plan.off_part) : nullptr;
    if (!encode_rows(&t.map_k64, k, d->Sq, d->B, 64) ||
        !encode_rows(&t.map_v64, v, d->Sq, d->B, 64) ||
        !encode_rows(&t.map_kh, k, d->Sq, d->B, 64, 2) ||
        !encode_rows(&t.map_qh, q, rows, d->B, 64, 2) ||
        !encode_rows(&t.map_doh, dout, rows, d->B, 64, 2) ||
        !encode_view(&t.map_pT, t.P, rows, plan.Skp / 64, d->B, pitch, 64, 2) ||
        !encode_view(&t.map_dsT, t.dS, rows, plan.Skp / 64, d->B, pitch, 64, 2) ||
        !encode_view(&t.map_ds, t.dS, rows, plan.Skp / 64, d->B, pitch, 128, 1) ||
        !encode_rows64b(&t.map_pw, t.P, plan.Skp, rows, d->B, pitch) ||
        !encode_rows64b(&t.map_dsw, t.dS, plan.Skp, rows, d->B, pitch))
      return PI_ERR_CUDA;
    t.ar = ar_mask; t.seg = segment_ids; t.mask_bs = d->mask_batch_stride;
    t.q = q; t.out = out; t.dout = dout; t.lse = lse;
    t.dq = dq; t.dk = dk; t.dv = dv;
    t.B = d->B; t.S = d->Sq; t.Hq = d->Hq; t.Skp = plan.Skp;
    t.n_chunks = plan.n_chunks; t.pairs_per_chunk = plan.pairs_per_chunk;
    t.clusters = plan.clusters;
    t.scale = d->softmax_scale;
    t.scale_log2 = d->softmax_scale * 1.4426950408889634f;
    return launched(launch_backward_tc(t, ctl, static_cast<cudaStream_t>(stream)));
  }
  BwdParams p;
  p.q = q; p.k = k; p.v = v; p.out = out; p.dout = dout; p.lse = lse;
  p.ar = ar_mask; p.seg = segment_ids; p.mask_bs = d->mask_batch_stride;
  p.dq = dq; p.dk = dk; p.dv = dv;
  p.codes = static_cast<uint32_t*>(workspace);
  const size_t codes_bytes = ((size_t)d->B * d->Sq * sizeof(uint32_t) + 255) & ~(size_t)255;
  p.D = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + codes_bytes);
  p.B = d->B; p.S = d->Sq; p.Hq = d->Hq; p.Hkv = d->Hkv; p.d = d->d;
  p.scale = d->softmax_scale;
  p.f32 = d->dtype == PI_F32;
  return launched(launch_backward(p, static_cast<cudaStream_t>(stream)));
}

int pi_attn_debug_mask(const pi_attn_desc* d, int mode, const uint8_t* ar_mask,
                       const int32_t* segment_ids, uint8_t* mask_out, pi_stream_t stream) {
  if (!d || !ar_mask || !mask_out) return PI_ERR_ARG;
  if (mode != 0 && mode != 1) return PI_ERR_ARG;
  if (d->B < 0 || d->Sq < 0 || d->P < 0) return PI_ERR_ARG;
  if (mode == 0 && d->P != 0) return PI_ERR_ARG;
  if (mode == 1 && segment_ids) return PI_ERR_ARG;
  if (d->mask_batch_stride < 0 || (d->mask_batch_stride != 0 && d->mask_batch_stride < d->Sq))
    return PI_ERR_ARG;
  if (d->Sq > kMaxTokens) return PI_ERR_UNSUPPORTED;
  if (d->B == 0 || d->Sq == 0) return PI_OK;
  return launched(launch_debug_mask(mode, d->B, d->Sq, d->P, ar_mask, segment_ids,
                                    d->mask_batch_stride, mask_out,
                                    static_cast<cudaStream_t>(stream)));
}

int pi_attn_debug_tiles(const pi_attn_desc* d, const uint8_t* ar_mask,
                        const int32_t* segment_ids, uint8_t* classes_out, pi_stream_t stream) {
  if (!d || !ar_mask || !classes_out) return PI_ERR_ARG;
  if (d->B < 0 || d->Sq < 0 || d->P != 0) return PI_ERR_ARG;
  if (d->mask_batch_stride < 0 || (d->mask_batch_stride != 0 && d->mask_batch_stride < d->Sq))
    return PI_ERR_ARG;
  if (d->Sq > kMaxTokens) return PI_ERR_UNSUPPORTED;
  if (!(d->Hq == 1 || d->Hq == 2 || d->Hq == 4 || d->Hq == 8 || d->Hq == 16))
    return PI_ERR_UNSUPPORTED;
  if (segment_ids && (reinterpret_cast<uintptr_t>(segment_ids) & 3u)) return PI_ERR_ALIGN;
  if (d->B == 0 || d->Sq == 0) return PI_OK;
  return launched(launch_debug_tiles(ar_mask, segment_ids, d->mask_batch_stride, d->B, d->Sq,
                                     d->Hq, classes_out, static_cast<cudaStream_t>(stream)));
}

int pi_attn_read_status(pi_stream_t stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PI_ERR_CUDA;
  int* p = status_ptr();
  if (!p) return PI_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PI_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return PI_ERR_CUDA;
  return v;
}

const char* pi_attn_status_string(int s) {
  switch (s) {
    case PI_OK: return "PI_OK";
    case PI_ERR_ARG: return "PI_ERR_ARG: invalid argument";
    case PI_ERR_ALIGN: return "PI_ERR_ALIGN: pointer not 16-byte aligned";
    case PI_ERR_UNSUPPORTED: return "PI_ERR_UNSUPPORTED: dtype or geometry not supported";
    case PI_ERR_CUDA: return "PI_ERR_CUDA: CUDA launch or runtime call failed";
    case PI_ERR_TIMEOUT: return "PI_ERR_TIMEOUT: a device-side bounded wait ran out";
    default: return "unknown pi_attn status";
  }
}

uint64_t pi_attn_set_wait_limit(uint64_t cycles) {
  return g_wait_limit.exchange(cycles ? cycles : kDefaultWaitLimit);
}

int pi_attn_selftest_wait(pi_stream_t stream) {
  DevCtl ctl;
  if (!make_ctl(&ctl)) return PI_ERR_CUDA;
  return launched(launch_selftest_wait(ctl, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

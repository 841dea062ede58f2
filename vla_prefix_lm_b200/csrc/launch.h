// launch.h -- internal launchers behind the C ABI (host side, not exported).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"

namespace piattn {

// Launches `kernel` so that it may begin while the previous kernel in `st` is
// still running (programmatic stream serialization): the kernel must call
// pdl_wait() before its first global memory access (common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Inputs of the fp32 SIMT path (both modes).  Prefill: k/v hold the S keys,
// kc/vc are null and P = 0.  Suffix: k/v hold the Sq suffix keys and kc/vc the
// P cached prefix keys.
struct SimtParams {
  const float* q;
  const float* k;
  const float* v;
  const float* kc;
  const float* vc;
  const uint8_t* ar;
  const int32_t* seg;
  long long mask_bs;
  float* out;
  float* lse;
  const uint8_t* cache_valid;  // suffix mode: [B, P] nonzero = valid cached key; may be null
  int B, Sq, P, Hq, Hkv, d;
  float scale;
};

cudaError_t launch_simt_f32(const SimtParams& p, const DevCtl& ctl, cudaStream_t st);

cudaError_t launch_debug_mask(int mode, int B, int Sq, int P, const uint8_t* ar,
                              const int32_t* seg, long long mask_bs, uint8_t* out,
                              cudaStream_t st);

cudaError_t launch_selftest_wait(const DevCtl& ctl, cudaStream_t st);

// Tile classes of the bf16 prefill kernel (tests): out [B][ceil(S*Hq/256)][ceil(S/128)].
cudaError_t launch_debug_tiles(const uint8_t* ar, const int32_t* seg, long long mask_bs, int B,
                               int S, int Hq, uint8_t* out, cudaStream_t st);

// Rotary embedding of q (and k) in place at positions cumsum(tmask) - 1
// (+ the valid prefix count when pmask is given).
struct RopeParams {
  void* q;
  void* k;                 // may be null
  const uint8_t* tmask;
  long long tmask_bs;
  const uint8_t* pmask;    // may be null
  long long pmask_bs;
  int32_t* pos_out;        // may be null
  int B, S, P, Hq, Hkv, d;
  float base;
  bool f32;
};

// Gradient of the prefill attention (backward.cu).
struct BwdParams {
  const void* q; const void* k; const void* v; const void* out; const void* dout;
  const float* lse;
  const uint8_t* ar; const int32_t* seg; long long mask_bs;
  float* dq; float* dk; float* dv;
  uint32_t* codes;                 // workspace: [B, S] packed mask codes
  float* D;                        // workspace: [B, S, Hq] rowsum(dO * O)
  int B, S, Hq, Hkv, d;
  float scale;
  bool f32;
};
size_t bwd_workspace_bytes(int B, int S, int Hq);
cudaError_t launch_backward(const BwdParams& p, cudaStream_t st);

// Gradient of the prefill on tensor cores (bwd_tc.cu): bf16, Hkv = 1, d = 256.
// Tensor maps are 4-D views (64, rows, column blocks, B) as for TcParams.
struct BwdTcParams {
  CUtensorMap map_k64;  // keys [B, S, 256], box (64, 64, 4, 1): the score pass's K item
  CUtensorMap map_v64;  // values, box (64, 64, 4, 1)
  CUtensorMap map_kh;   // keys, box (64, 64, 2, 1): 64 keys x 128 columns
  CUtensorMap map_qh;   // q rows, box (64, 64, 2, 1)
  CUtensorMap map_doh;  // dout rows, box (64, 64, 2, 1)
  CUtensorMap map_pT;   // P workspace [B, S*Hq, Skp] as (64, rows, Skp/64, B), box (64, 64, 2, 1)
  CUtensorMap map_dsT;  // dS workspace, box (64, 64, 2, 1)
  CUtensorMap map_ds;   // dS workspace, box (64, 128, 1, 1)
  CUtensorMap map_pw;   // P workspace as (Skp, S*Hq, B), box (32, 32, 1), 64-byte swizzle
  CUtensorMap map_dsw;  // dS workspace, the same view (the score pass's stores)
  const uint8_t* ar;
  const int32_t* seg;
  long long mask_bs;
  const void* q;        // q rows (bf16), for the score pass's TMEM copy
  const void* out;      // forward output (bf16), for D
  const void* dout;
  const float* lse;     // [B, S*Hq] natural log
  float* D;             // workspace [B, S*Hq]
  __nv_bfloat16* P;     // workspace [B, S*Hq, Skp]
  __nv_bfloat16* dS;    // workspace [B, S*Hq, Skp]
  float* part;          // workspace: dK/dV partials per row chunk (n_chunks > 1)
  float* dq;
  float* dk;
  float* dv;
  int B, S, Hq, Skp, n_chunks, pairs_per_chunk;
  int clusters;         // SM pairs the persistent passes use
  float scale, scale_log2;
};

// Sizes of the tensor-core backward for a shape: row tiles, key groups, the
// padded key count of the P / dS workspace, the dK/dV row chunks, and the
// workspace layout (byte offsets, total).
struct BwdTcPlan {
  int n_pairs, n_sup, Skp, n_chunks, pairs_per_chunk, clusters;
  size_t off_D, off_P, off_dS, off_part, bytes;
};
BwdTcPlan bwd_tc_plan(int B, int S, int Hq, int sms);
cudaError_t launch_backward_tc(const BwdTcParams& p, const DevCtl& ctl, cudaStream_t st);
int sm_count();

cudaError_t launch_rope(const RopeParams& p, const DevCtl& ctl, cudaStream_t st);
// Shared memory one RoPE CTA may use: (Hq + Hkv) * d * element size must fit.
size_t rope_max_smem();

// x (fp32) += dt * v (bf16 or fp32), n elements.
cudaError_t launch_euler(float* x, const void* v, bool v_f32, float dt, long long n,
                         cudaStream_t st);

// bf16 tcgen05 path.  All tensors are [B, tokens, heads, 256] bf16; maps are
// encoded by the ABI layer.
struct TcParams {
  // 4-D views (64, rows, 4 column blocks, B) of [B, rows, 256] bf16 tensors
  CUtensorMap map_q;    // q rows (Sq*Hq per batch), box (64, 128, 4, 1)
  CUtensorMap map_k;    // keys (prefill: S; suffix: Sq), 64 keys x 256: box (64, 64, 4, 1)
  CUtensorMap map_kc;   // suffix mode: cached keys (P per batch); unused in prefill
  CUtensorMap map_o;    // out rows, box (64, 32, 1, 1): one 64-column block
  CUtensorMap map_vh;   // values, 64 keys x 128 columns: box (64, 64, 2, 1)
  CUtensorMap map_vch;  // cached values, same box
  const uint8_t* ar;
  const int32_t* seg;
  long long mask_bs;
  float* lse;           // prefill only; may be null
  const uint8_t* cache_valid;  // suffix mode: [B, P] nonzero = valid cached key; may be null
  float* ws;            // split-K partials (suffix mode); may be null
  void* out_ptr;        // bf16 output rows (written by the combine kernel under split-K)
  int B, Sq, P, Hq;
  int n_splits;         // KV splits per query tile (1 = write final output)
  // Prefill tail split: units [0, n_main) run whole (full rounds of the
  // clusters); each later unit runs as tail_splits pieces whose fp32 partials
  // go to ws ([piece][256 rows] O, then (m, l)) and tail_combine_kernel merges.
  int n_main;           // B * query tiles when there is no tail split
  int tail_splits;      // 1: no tail split
  float scale_log2;     // softmax_scale * log2(e)
  float scale;          // softmax_scale
};

// CTA-pair (2-SM) form: 256 query rows per cluster of 2, 128-key tiles.  With
// p.n_splits > 1 the key tiles are split over that many pairs per query tile,
// partials go to p.ws and a combine kernel writes the output.
cudaError_t launch_tc_pair(const TcParams& p, bool suffix_mode, const DevCtl& ctl,
                           cudaStream_t st);

size_t tc_suffix_workspace_bytes(int B, int Sq, int P, int Hq);

// Scratch of the prefill tail split on the current device: at most one round
// of pieces (one per SM pair) of 256 rows, fp32 O and (m, l).
size_t tc_prefill_tail_bytes();
// Pieces per tail unit the prefill splits its last round into (1: none).
int tc_prefill_tail_splits(int B, int Sq, int Hq);
int tc_suffix_splits(int B, int Sq, int P, int Hq);

// Merges split partials (unnormalised O [splits][rows][256] fp32, then (m, l)
// [splits][rows][2] in the exp2 domain) into bf16 rows.
cudaError_t launch_combine(const float* ws, __nv_bfloat16* out, int n_splits, long long n_rows,
                           cudaStream_t st);

// Suffix pass with at most 8 query rows per batch element (decode.cu): bf16,
// one KV head, d = 256.  Needs no workspace.  Cache and suffix K/V as 4-D
// views, box (64, kDecodeTileKeys, 4, 1).
constexpr int kDecodeTileKeys = 16;
struct DecodeParams {
  CUtensorMap map_kc;
  CUtensorMap map_vc;
  CUtensorMap map_k;
  CUtensorMap map_v;
  const __nv_bfloat16* q;       // [B, Sq, Hq, 256]
  const uint8_t* ar;            // suffix ar_mask rows
  const int32_t* seg;           // suffix segment ids (may be null)
  long long mask_bs;
  const uint8_t* cache_valid;   // [B, P] (may be null)
  __nv_bfloat16* out;
  int B, Sq, P, Hq;
  float scale_log2;
};
bool decode_applies(int Sq, int Hq);
cudaError_t launch_decode(const DecodeParams& p, const DevCtl& ctl, cudaStream_t st);

}  // namespace piattn

// mask.cuh -- the in-kernel visibility predicate of the prefix-LM joint
// attention, shared by every kernel of the library (and by the debug-mask
// export that tests compare bit for bit with an explicitly built mask).
//
// Rule ("π0.5 vs MM-DiT joint attention", section π0.5:三段,两处看不到):
//   key j is visible to query i  iff  cs[j] <= cs[i]
//                                 and not (seg[i] == EXPERT and seg[j] == FAST)
// with cs = inclusive cumsum of the boolean ar_mask over the token axis.
// Suffix-only pass ("VLA 代码精读 - OpenPI & StarVLA", 1.6): cached prefix
// keys are visible to every suffix query; suffix keys follow the rule over the
// suffix tokens alone.
//
// Encoding.  Each token carries one packed code:
//     code = (cs << 2) | (is_expert << 1) | is_fast
// so that   visible(cq, ck) = (ck >> 2) <= (cq >> 2) && !((cq & 2) && (ck & 1)).
// Cached prefix keys get code 0, which every query code admits.  cs <= S, so
// S <= 16383 keeps a code within 16 bits.
#pragma once
#include <cstdint>

namespace piattn {

constexpr int kSegFast = 1;
constexpr int kSegExpert = 2;
constexpr int kMaxTokens = 16383;

__host__ __device__ __forceinline__ uint32_t make_code(uint32_t cs, int seg) {
  return (cs << 2) | (seg == kSegExpert ? 2u : 0u) | (seg == kSegFast ? 1u : 0u);
}

__host__ __device__ __forceinline__ bool visible(uint32_t cq, uint32_t ck) {
  return (ck >> 2) <= (cq >> 2) && !((cq & 2u) && (ck & 1u));
}

// Block-wide inclusive scan of (ar != 0) over one batch row of S tokens,
// written as packed codes into `codes` (shared or global).  Every thread of
// the block must call it.  `scratch` is shared memory for at least 33 ints.
// Tokens are visited in chunks of blockDim.x; lanes scan with shuffles, warp
// totals are scanned by warp 0, and a running carry crosses the chunks.
template <typename CodeT>
__device__ void build_codes(const uint8_t* __restrict__ ar, const int32_t* __restrict__ seg,
                            int S, CodeT* codes, int* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  if (threadIdx.x == 0) scratch[32] = 0;
  __syncthreads();
  for (int base = 0; base < S; base += blockDim.x) {
    const int t = base + threadIdx.x;
    int x = (t < S && ar[t] != 0) ? 1 : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = lane < nwarps ? scratch[lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += y;
      }
      if (lane < nwarps) scratch[lane] = w;  // inclusive warp prefix
    }
    __syncthreads();
    const int carry = scratch[32];
    const int cs = carry + x + (warp > 0 ? scratch[warp - 1] : 0);
    if (t < S) codes[t] = (CodeT)make_code((uint32_t)cs, seg ? seg[t] : 0);
    __syncthreads();
    if (threadIdx.x == 0) scratch[32] = carry + scratch[nwarps - 1];
    __syncthreads();
  }
}

}  // namespace piattn

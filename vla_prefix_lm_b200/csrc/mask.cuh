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
// Padding (not in the pages' workloads; openpi and Pi0-FAST AND a per-token
// validity mask into the attention mask): a negative segment id marks a
// padding token, which no query reads and which reads no key.
//
// Encoding.  Each token carries one packed code:
//     code = (cs << 2) | (is_expert << 1) | is_fast,   padding: both flag bits
// so that   visible(cq, ck) = neither is padding
//                             && (ck >> 2) <= (cq >> 2) && !((cq & 2) && (ck & 1)).
// (Padding keys also carry the FAST bit, so the expert rule alone already
// hides them from expert queries.)  Cached prefix keys get code 0, which every
// non-padding query admits.  cs <= S, so S <= 16383 keeps a code in 16 bits.
#pragma once
#include <cstdint>

namespace piattn {

constexpr int kSegFast = 1;
constexpr int kSegExpert = 2;
constexpr int kMaxTokens = 16383;

__host__ __device__ __forceinline__ uint32_t make_code(uint32_t cs, int seg) {
  if (seg < 0) return (cs << 2) | 3u;
  return (cs << 2) | (seg == kSegExpert ? 2u : 0u) | (seg == kSegFast ? 1u : 0u);
}

__host__ __device__ __forceinline__ bool is_pad(uint32_t code) { return (code & 3u) == 3u; }

__host__ __device__ __forceinline__ bool visible(uint32_t cq, uint32_t ck) {
  return !is_pad(cq) && !is_pad(ck) && (ck >> 2) <= (cq >> 2) && !((cq & 2u) && (ck & 1u));
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

// Same result as build_codes, for the tensor-core kernel.  Each thread owns
// 32 consecutive tokens per round: their ar_mask bytes (and segment ids) are
// all loaded up front -- 16-byte vectors when aligned -- and reduced to
// 32-bit masks; one shuffle scan across the warp and a short scan over the
// kThreads/32 warp totals give each thread its starting block index.  Codes
// past S up to S_pad (a multiple of 32) are 0xFFFF.  `scratch` is shared
// memory for kThreads/32 ints.  Every thread of the block must call it; it
// ends with a block barrier.
__device__ __forceinline__ uint32_t nonzero_byte_bits(uint32_t w) {
  return ((w & 0xFFu) ? 1u : 0u) | ((w & 0xFF00u) ? 2u : 0u) | ((w & 0xFF0000u) ? 4u : 0u) |
         ((w & 0xFF000000u) ? 8u : 0u);
}

// The ar_mask bits and segment flags of 32 consecutive tokens starting at t0
// (16-byte vector loads when aligned).  Tokens at or past S read as False / 0.
// A padding token sets both its fast and its expert bit.
struct Flags32 {
  uint32_t bits, fast, expert;
};

__device__ __forceinline__ Flags32 load_flags32(const uint8_t* __restrict__ ar,
                                                const int32_t* __restrict__ seg, int S, int t0) {
  Flags32 f{0u, 0u, 0u};
  if (t0 >= S) return f;
  if (t0 + 32 <= S && (reinterpret_cast<uintptr_t>(ar + t0) & 15u) == 0) {
    const uint4 a = *reinterpret_cast<const uint4*>(ar + t0);
    const uint4 c = *reinterpret_cast<const uint4*>(ar + t0 + 16);
    f.bits = nonzero_byte_bits(a.x) | (nonzero_byte_bits(a.y) << 4) |
             (nonzero_byte_bits(a.z) << 8) | (nonzero_byte_bits(a.w) << 12) |
             (nonzero_byte_bits(c.x) << 16) | (nonzero_byte_bits(c.y) << 20) |
             (nonzero_byte_bits(c.z) << 24) | (nonzero_byte_bits(c.w) << 28);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (t0 + i < S && ar[t0 + i] != 0) f.bits |= 1u << i;
  }
  if (seg != nullptr) {
    if (t0 + 32 <= S && (reinterpret_cast<uintptr_t>(seg + t0) & 15u) == 0) {
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const int4 v = reinterpret_cast<const int4*>(seg + t0)[g];
        const int sv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          f.fast |= (sv[h] == kSegFast || sv[h] < 0 ? 1u : 0u) << (4 * g + h);
          f.expert |= (sv[h] == kSegExpert || sv[h] < 0 ? 1u : 0u) << (4 * g + h);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int sv = t0 + i < S ? seg[t0 + i] : 0;
        f.fast |= (sv == kSegFast || sv < 0 ? 1u : 0u) << i;
        f.expert |= (sv == kSegExpert || sv < 0 ? 1u : 0u) << i;
      }
    }
  }
  return f;
}

// Same result as build_codes, for the tensor-core kernels.  Each thread owns
// 32 consecutive tokens per round (their flags come from load_flags32; the
// first round's may be loaded early by the caller and passed in `first`); one
// shuffle scan across the warp and a short scan over the kThreads/32 warp
// totals give each thread its starting block index.  Codes past S up to S_pad
// (a multiple of 32) are 0xFFFF.  `scratch` is shared memory for kThreads/32
// ints.  Every thread of the block must call it; it ends with a block barrier.
// Per-128-token summaries the tile classifier needs: the block index (cs) of
// the tile's first token, the largest cs in it, and whether it holds any /
// only FAST tokens (padding counts as FAST there), and whether it holds any /
// only padding tokens.
struct TileSums {
  uint16_t* cs_first;
  uint16_t* cs_last;
  uint8_t* fast;   // bit 0: any FAST, bit 1: all FAST, bit 2: any padding, bit 3: all padding
};

template <int kThreads>
__device__ void build_codes_x32(const uint8_t* __restrict__ ar, const int32_t* __restrict__ seg,
                                int S, int S_pad, uint16_t* codes, int* scratch,
                                Flags32 first, TileSums sums) {
  constexpr int kWarps = kThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int carry = 0;
  for (int base = 0; base < S_pad; base += kThreads * 32) {
    const int t0 = base + (int)threadIdx.x * 32;
    const Flags32 f = base == 0 ? first : load_flags32(ar, seg, S, t0);
    const int cnt = __popc(f.bits);
    int x = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int v = scratch[w];
      before += (w < warp) ? v : 0;
      total += v;
    }
    const int excl = carry + before + x - cnt;  // tokens before t0 that are True
    if (t0 < S_pad) {
      uint32_t packed[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        uint32_t c2[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int k = i + h;
          const uint32_t upto = k == 31 ? 0xFFFFFFFFu : ((2u << k) - 1u);
          const uint32_t cs = (uint32_t)excl + (uint32_t)__popc(f.bits & upto);
          c2[h] = t0 + k < S
                      ? ((cs << 2) | (((f.expert >> k) & 1u) << 1) | ((f.fast >> k) & 1u))
                      : 0xFFFFu;
        }
        packed[i / 2] = c2[0] | (c2[1] << 16);
      }
      uint4* dst = reinterpret_cast<uint4*>(codes + t0);   // t0 is a multiple of 32
#pragma unroll
      for (int g = 0; g < 4; ++g)
        dst[g] = make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
    }
    if (sums.cs_first != nullptr) {
      // Four consecutive lanes own one 128-token tile: combine their parts.
      const int nv = min(max(S - t0, 0), 32);                 // valid tokens here
      const uint32_t vmask = nv >= 32 ? 0xFFFFFFFFu : ((1u << nv) - 1u);
      const uint32_t pad = f.fast & f.expert;
      uint32_t any_f = (f.fast & vmask) != 0u ? 1u : 0u;
      uint32_t all_f = (f.fast & vmask) == vmask ? 1u : 0u;   // vacuous when nv == 0
      uint32_t any_p = (pad & vmask) != 0u ? 1u : 0u;
      uint32_t all_p = (pad & vmask) == vmask ? 1u : 0u;
      uint32_t cs_hi = nv > 0 ? (uint32_t)excl + (uint32_t)__popc(f.bits & vmask) : 0u;
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        any_f |= __shfl_xor_sync(0xffffffffu, any_f, off);
        all_f &= __shfl_xor_sync(0xffffffffu, all_f, off);
        any_p |= __shfl_xor_sync(0xffffffffu, any_p, off);
        all_p &= __shfl_xor_sync(0xffffffffu, all_p, off);
        cs_hi = max(cs_hi, __shfl_xor_sync(0xffffffffu, cs_hi, off));
      }
      if ((lane & 3) == 0 && t0 < S) {
        const int tile = t0 >> 7;
        sums.cs_first[tile] = (uint16_t)((uint32_t)excl + (f.bits & 1u));
        sums.cs_last[tile] = (uint16_t)cs_hi;
        sums.fast[tile] = (uint8_t)(any_f | (all_f << 1) | (any_p << 2) | (all_p << 3));
      }
    }
    carry += total;
    __syncthreads();
  }
}

}  // namespace piattn

// simt.cu -- fp32 attention on CUDA cores (both modes), the debug-mask
// export, and the bounded-wait self-test.
//
// The fp32 path exists for the fp32 workloads, whose 1e-4 tolerance rules out
// TF32 tensor-core arithmetic: it is a plain online-softmax loop with one warp
// per (batch, query token, query head) row, q and the running output held in
// registers (d/32 per lane), scores reduced with warp shuffles.  The mask is
// the shared predicate of mask.cuh evaluated per (query, key) pair.
#include <cfloat>

#include "launch.h"
#include "mask.cuh"

namespace piattn {

namespace {

constexpr int kSimtThreads = 256;
constexpr int kSimtTokensPerBlock = 8;

template <int D>
__global__ void __launch_bounds__(kSimtThreads)
    simt_attention_f32(const SimtParams p) {
  extern __shared__ uint32_t s_codes[];  // [Sq] codes of the query / suffix tokens
  __shared__ int s_scan[33];
  constexpr int C = D / 32;
  const int b = blockIdx.y;
  const uint8_t* ar = p.ar + (long long)b * p.mask_bs;
  const int32_t* seg = p.seg ? p.seg + (long long)b * p.mask_bs : nullptr;
  build_codes<uint32_t>(ar, seg, p.Sq, s_codes, s_scan);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tok0 = blockIdx.x * kSimtTokensPerBlock;
  const int ntok = min(kSimtTokensPerBlock, p.Sq - tok0);
  const int group = p.Hq / p.Hkv;
  const int Sk = p.P + p.Sq;

  for (int r = warp; r < ntok * p.Hq; r += kSimtThreads / 32) {
    const int i = tok0 + r / p.Hq, h = r % p.Hq, g = h / group;
    const float* qrow = p.q + (((long long)b * p.Sq + i) * p.Hq + h) * D;
    float qv[C], acc[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
      qv[c] = qrow[lane + 32 * c] * p.scale;
      acc[c] = 0.f;
    }
    const uint32_t cq = s_codes[i];
    float m = -FLT_MAX, l = 0.f;
    for (int j = 0; j < Sk; ++j) {
      const float* krow;
      const float* vrow;
      if (j < p.P) {  // cached prefix key: visible to every valid suffix query
        if (is_pad(cq) || (p.cache_valid && p.cache_valid[(long long)b * p.P + j] == 0)) continue;
        krow = p.kc + (((long long)b * p.P + j) * p.Hkv + g) * D;
        vrow = p.vc + (((long long)b * p.P + j) * p.Hkv + g) * D;
      } else {
        const int js = j - p.P;
        if (!visible(cq, s_codes[js])) continue;
        krow = p.k + (((long long)b * p.Sq + js) * p.Hkv + g) * D;
        vrow = p.v + (((long long)b * p.Sq + js) * p.Hkv + g) * D;
      }
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < C; ++c) s = fmaf(qv[c], krow[lane + 32 * c], s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      const float m_new = fmaxf(m, s);
      const float corr = expf(m - m_new);
      const float e = expf(s - m_new);
      l = l * corr + e;
#pragma unroll
      for (int c = 0; c < C; ++c) acc[c] = fmaf(acc[c], corr, e * vrow[lane + 32 * c]);
      m = m_new;
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;   // no visible key (padding): 0
    float* orow = p.out + (((long long)b * p.Sq + i) * p.Hq + h) * D;
#pragma unroll
    for (int c = 0; c < C; ++c) orow[lane + 32 * c] = acc[c] * inv;
    if (p.lse && lane == 0)
      p.lse[((long long)b * p.Sq + i) * p.Hq + h] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

__global__ void __launch_bounds__(256)
    debug_mask_kernel(int mode, int Sq, int P, const uint8_t* ar_all, const int32_t* seg_all,
                      long long mask_bs, uint8_t* out) {
  extern __shared__ uint32_t s_codes[];
  __shared__ int s_scan[33];
  const int b = blockIdx.y;
  const uint8_t* ar = ar_all + (long long)b * mask_bs;
  const int32_t* seg = seg_all ? seg_all + (long long)b * mask_bs : nullptr;
  build_codes<uint32_t>(ar, seg, Sq, s_codes, s_scan);
  const int Sk = mode == 0 ? Sq : P + Sq;
  const int i0 = blockIdx.x * 8;
  for (int i = i0; i < min(i0 + 8, Sq); ++i) {
    const uint32_t cq = s_codes[i];
    uint8_t* row = out + ((long long)b * Sq + i) * Sk;
    for (int j = threadIdx.x; j < Sk; j += blockDim.x) {
      bool vis;
      if (mode == 0) {
        vis = visible(cq, s_codes[j]);
      } else {
        vis = j < P ? visible(cq, 0u) : visible(cq, s_codes[j - P]);
      }
      row[j] = vis ? 1 : 0;
    }
  }
}

__global__ void selftest_wait_kernel(DevCtl ctl) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing arrives on `bar`: the bounded wait must run out and report it.
    (void)mbar_wait(&bar, 0, ctl);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_simt_f32(const SimtParams& p, const DevCtl& ctl, cudaStream_t st) {
  (void)ctl;
  dim3 grid((p.Sq + kSimtTokensPerBlock - 1) / kSimtTokensPerBlock, p.B);
  const size_t smem = sizeof(uint32_t) * (size_t)p.Sq;
  auto launch = [&](auto kern) -> cudaError_t {
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
    }
    kern<<<grid, kSimtThreads, smem, st>>>(p);
    return cudaGetLastError();
  };
  switch (p.d) {
    case 32: return launch(simt_attention_f32<32>);
    case 64: return launch(simt_attention_f32<64>);
    case 128: return launch(simt_attention_f32<128>);
    case 256: return launch(simt_attention_f32<256>);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_debug_mask(int mode, int B, int Sq, int P, const uint8_t* ar,
                              const int32_t* seg, long long mask_bs, uint8_t* out,
                              cudaStream_t st) {
  dim3 grid((Sq + 7) / 8, B);
  const size_t smem = sizeof(uint32_t) * (size_t)Sq;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(debug_mask_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  debug_mask_kernel<<<grid, 256, smem, st>>>(mode, Sq, P, ar, seg, mask_bs, out);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(const DevCtl& ctl, cudaStream_t st) {
  selftest_wait_kernel<<<1, 32, 0, st>>>(ctl);
  return cudaGetLastError();
}

}  // namespace piattn

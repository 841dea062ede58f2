// prepost.cu -- the steps on either side of the attention: rotary position
// embedding of q and k at the pages' positions, and the Euler update of the
// flow-matching sampler.
//
// Sources ("VLA 代码精读 - OpenPI & StarVLA", 1.5 and 1.6): positions are
// cumsum(mask) - 1 over the tokens of a call, and a suffix pass continues
// after the valid prefix tokens (sum(prefix_mask) + cumsum(suffix_mask) - 1);
// the sampler steps x <- x + dt * v.  The pages name the LLM's built-in RoPE
// without a formula: here the standard rotation of (i, i + d/2) pairs by
// pos * base^(-2i/d).
//
// Both kernels are HBM-bound elementwise passes.
//
// RoPE: one CTA per (batch, run of tokens); a thread owns one (token, 16-byte
// column slice of the first half of the head) and the matching slice of the
// second half.  The CTA first forms its tokens' positions (a block count of
// the mask bytes before the run -- and of the valid prefix tokens -- plus one
// ballot over the run's own bytes) and the inverse frequencies
// base^(-2i/d) in fp64.  Each thread then forms its slice's angles once (the
// product pos * inv_freq reduced modulo 2*pi in fp64, so that positions in
// the thousands keep fp32 accuracy, then sincosf) and rotates that slice of
// every head of q and k in place, straight from and to global memory: each
// warp access is a contiguous run of 16-byte vectors, and with the heads'
// loads issued together many requests are in flight per SM, which the pass
// needs to stream at HBM rate.  (A form that staged each run through
// shared memory with one bulk copy per CTA kept DRAM at a fifth of its
// bandwidth: too few bytes in flight per SM.)
#include <algorithm>
#include <cstdint>

#include "launch.h"

namespace piattn {

namespace {

constexpr int kRopeThreads = 128;
constexpr int kRopeMaxTok = 32;                  // one ballot covers a CTA's tokens
constexpr int kRopeMaxSmem = 160 * 1024;         // bound on one token's heads (ABI limit)

template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> { static constexpr int N = 8; };   // 16 B
template <> struct Vec<float> { static constexpr int N = 4; };           // 16 B

__device__ __forceinline__ void unpack(const uint4& u, float (&f)[8], __nv_bfloat16*) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ uint4 pack(const float (&f)[8], __nv_bfloat16*) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}
__device__ __forceinline__ void unpack(const uint4& u, float (&f)[4], float*) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ uint4 pack(const float (&f)[4], float*) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}

// kU heads' loads are in flight together per thread; kMinBlocks CTAs of the
// kernel fit on an SM.  A grid that fills the GPU several times over keeps
// four heads in flight and five CTAs per SM; a grid of at most two CTAs per
// SM takes all nine heads of the pi0 shapes at once, four CTAs per SM.
template <typename T, int kU, int kMinBlocks>
__global__ void __launch_bounds__(kRopeThreads, kMinBlocks)
    rope_kernel(T* q, T* k, const uint8_t* tmask, long long tmask_bs, const uint8_t* pmask,
                long long pmask_bs, int S, int P, int Hq, int Hkv, int d, int tok,
                double log2_base, int32_t* pos_out) {
  constexpr int N = Vec<T>::N;
  __shared__ double s_inv[128];                 // base^(-2i/d), i < d/2 <= 128
  __shared__ int s_count[kRopeThreads / 32];
  __shared__ uint32_t s_bits;
  pdl_wait();                                   // q and k may come from the kernel before
  pdl_launch_dependents();
  const int b = blockIdx.y;
  const int t0 = blockIdx.x * tok;
  const int nt = min(tok, S - t0);
  const int half = d / 2;
  const int vpr = half / N;                     // vectors per half row
  const int Hk = k ? Hkv : 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // Positions: valid tokens before the run (and valid prefix tokens) by a
  // block count, the run's own mask bits by one ballot.
  const uint8_t* tm = tmask + (long long)b * tmask_bs;
  int cnt = 0;
  for (int t = threadIdx.x * 4; t < t0; t += kRopeThreads * 4) {
#pragma unroll
    for (int e = 0; e < 4; ++e) cnt += (t + e < t0 && tm[t + e] != 0) ? 1 : 0;
  }
  if (pmask) {
    const uint8_t* pm = pmask + (long long)b * pmask_bs;
    for (int t = threadIdx.x * 4; t < P; t += kRopeThreads * 4) {
#pragma unroll
      for (int e = 0; e < 4; ++e) cnt += (t + e < P && pm[t + e] != 0) ? 1 : 0;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  if (lane == 0) s_count[warp] = cnt;
  if (warp == 0) {
    const uint32_t bits = __ballot_sync(0xffffffffu, lane < nt && tm[t0 + lane] != 0);
    if (lane == 0) s_bits = bits;
  }
  for (int i = threadIdx.x; i < half; i += kRopeThreads)
    s_inv[i] = exp2(-2.0 * (double)i / (double)d * log2_base);
  __syncthreads();
  int base = -1;
#pragma unroll
  for (int w = 0; w < kRopeThreads / 32; ++w) base += s_count[w];
  const uint32_t bits = s_bits;

  const int tl = threadIdx.x / vpr, vi = threadIdx.x % vpr;
  if (tl >= nt) return;
  const int pos = base + __popc(bits & (0xFFFFFFFFu >> (31 - tl)));
  const long long bt = (long long)b * S + t0 + tl;
  if (pos_out && vi == 0) pos_out[bt] = pos;
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  float cs[N], sn[N];
#pragma unroll
  for (int e = 0; e < N; ++e) {
    double ang = (double)pos * s_inv[vi * N + e];
    ang -= two_pi * rint(ang * inv_two_pi);
    sincosf((float)ang, &sn[e], &cs[e]);
  }
  T* gq = q + bt * Hq * d + vi * N;
  T* gk = k ? k + bt * Hkv * d + vi * N : nullptr;
  for (int h0 = 0; h0 < Hq + Hk; h0 += kU) {
    uint4 x1[kU], x2[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int h = h0 + u;
      if (h < Hq + Hk) {
        T* row = h < Hq ? gq + (long long)h * d : gk + (long long)(h - Hq) * d;
        x1[u] = *reinterpret_cast<const uint4*>(row);
        x2[u] = *reinterpret_cast<const uint4*>(row + half);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int h = h0 + u;
      if (h < Hq + Hk) {
        T* row = h < Hq ? gq + (long long)h * d : gk + (long long)(h - Hq) * d;
        float a[N], c[N], o1[N], o2[N];
        unpack(x1[u], a, (T*)nullptr);
        unpack(x2[u], c, (T*)nullptr);
#pragma unroll
        for (int e = 0; e < N; ++e) {
          o1[e] = a[e] * cs[e] - c[e] * sn[e];
          o2[e] = c[e] * cs[e] + a[e] * sn[e];
        }
        *reinterpret_cast<uint4*>(row) = pack(o1, (T*)nullptr);
        *reinterpret_cast<uint4*>(row + half) = pack(o2, (T*)nullptr);
      }
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
    euler_kernel(float* __restrict__ x, const T* __restrict__ v, float dt, long long n) {
  pdl_wait();                                   // v comes from the attention pass before
  pdl_launch_dependents();
  const long long n4 = n / 4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 a = reinterpret_cast<float4*>(x)[i];
    float w[4];
    if constexpr (sizeof(T) == 2) {
      const uint2 u = reinterpret_cast<const uint2*>(v)[i];
      w[0] = __uint_as_float(u.x << 16); w[1] = __uint_as_float(u.x & 0xFFFF0000u);
      w[2] = __uint_as_float(u.y << 16); w[3] = __uint_as_float(u.y & 0xFFFF0000u);
    } else {
      const float4 u = reinterpret_cast<const float4*>(v)[i];
      w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
    }
    a.x = fmaf(dt, w[0], a.x); a.y = fmaf(dt, w[1], a.y);
    a.z = fmaf(dt, w[2], a.z); a.w = fmaf(dt, w[3], a.w);
    reinterpret_cast<float4*>(x)[i] = a;
  }
  // tail
  for (long long i = n4 * 4 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += stride) {
    float w;
    if constexpr (sizeof(T) == 2) {
      w = __bfloat162float(v[i]);
    } else {
      w = v[i];
    }
    x[i] = fmaf(dt, w, x[i]);
  }
}

}  // namespace

// Tokens per CTA: one thread per (token, 16-byte slice of a half row), at most
// 32 tokens (one ballot).
int rope_tokens_per_cta(int d, bool f32) {
  const int vpr = (d / 2) / (f32 ? 4 : 8);
  return std::max(1, std::min(kRopeMaxTok, kRopeThreads / std::max(vpr, 1)));
}

size_t rope_max_smem() { return kRopeMaxSmem; }

cudaError_t launch_rope(const RopeParams& p, const DevCtl& ctl, cudaStream_t st) {
  (void)ctl;   // no waits in this kernel
  const int tok = rope_tokens_per_cta(p.d, p.f32);
  dim3 grid((p.S + tok - 1) / tok, p.B);
  const double log2_base = log2((double)p.base);
  const bool small = (long long)grid.x * grid.y <= 2LL * sm_count();
  if (p.f32)
    return launch_pdl(small ? rope_kernel<float, 9, 4> : rope_kernel<float, 4, 5>, grid,
                      dim3(kRopeThreads), 0, st, static_cast<float*>(p.q),
                      static_cast<float*>(p.k), p.tmask, p.tmask_bs, p.pmask, p.pmask_bs, p.S,
                      p.P, p.Hq, p.Hkv, p.d, tok, log2_base, p.pos_out);
  return launch_pdl(small ? rope_kernel<__nv_bfloat16, 9, 4> : rope_kernel<__nv_bfloat16, 4, 5>,
                    grid, dim3(kRopeThreads), 0, st, static_cast<__nv_bfloat16*>(p.q),
                    static_cast<__nv_bfloat16*>(p.k), p.tmask, p.tmask_bs, p.pmask, p.pmask_bs,
                    p.S, p.P, p.Hq, p.Hkv, p.d, tok, log2_base, p.pos_out);
}

cudaError_t launch_euler(float* x, const void* v, bool v_f32, float dt, long long n,
                         cudaStream_t st) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long blocks_needed = (n / 4 + 255) / 256 + 1;
  const int grid = (int)std::min<long long>(blocks_needed, (long long)sms * 8);
  if (v_f32)
    return launch_pdl(euler_kernel<float>, dim3(grid), dim3(256), 0, st, x,
                      static_cast<const float*>(v), dt, n);
  return launch_pdl(euler_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, x,
                    static_cast<const __nv_bfloat16*>(v), dt, n);
}

}  // namespace piattn

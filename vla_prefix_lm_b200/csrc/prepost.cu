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
// Both kernels are HBM-bound elementwise passes.  RoPE: one CTA per (batch,
// 32-token chunk); the chunk's positions come from a block count of the mask
// bytes before it plus a warp scan inside it, the angles are formed and
// reduced modulo 2*pi in fp64 (so large positions keep fp32-level accuracy),
// their sine and cosine are tabulated in shared memory once per (token, pair)
// and applied to every head with 16-byte vector loads and stores.
#include <cstdint>

#include "launch.h"

namespace piattn {

namespace {

constexpr int kRopeTokens = 32;
constexpr int kRopeThreads = 256;

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

// Rotates the heads of one tensor [B, S, H, d] for the chunk's tokens.
template <typename T>
__device__ void rope_rows(T* x, int H, int d, int S, int b, int t0, int nt, const float* cs,
                          const float* sn) {
  constexpr int N = Vec<T>::N;
  const int half = d / 2;
  const int vpr = half / N;                     // vectors per half row
  const int total = nt * H * vpr;
  for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
    const int vi = idx % vpr;
    const int h = (idx / vpr) % H;
    const int tl = idx / (vpr * H);
    T* row = x + (((long long)b * S + t0 + tl) * H + h) * d;
    uint4* p1 = reinterpret_cast<uint4*>(row + vi * N);
    uint4* p2 = reinterpret_cast<uint4*>(row + half + vi * N);
    float a[N], c[N];
    unpack(*p1, a, (T*)nullptr);
    unpack(*p2, c, (T*)nullptr);
    const float* ct = cs + tl * half + vi * N;
    const float* st = sn + tl * half + vi * N;
    float o1[N], o2[N];
#pragma unroll
    for (int e = 0; e < N; ++e) {
      o1[e] = a[e] * ct[e] - c[e] * st[e];
      o2[e] = c[e] * ct[e] + a[e] * st[e];
    }
    *p1 = pack(o1, (T*)nullptr);
    *p2 = pack(o2, (T*)nullptr);
  }
}

template <typename T>
__global__ void __launch_bounds__(kRopeThreads)
    rope_kernel(T* q, T* k, const uint8_t* tmask, long long tmask_bs, const uint8_t* pmask,
                long long pmask_bs, int S, int P, int Hq, int Hkv, int d, double log2_base,
                int32_t* pos_out) {
  extern __shared__ float tab[];                // cos [32][d/2] | sin [32][d/2]
  __shared__ int s_count[kRopeThreads / 32];
  __shared__ int s_pos[kRopeTokens];
  const int b = blockIdx.y;
  const int t0 = blockIdx.x * kRopeTokens;
  const int nt = min(kRopeTokens, S - t0);
  const int half = d / 2;
  const uint8_t* tm = tmask + (long long)b * tmask_bs;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // Valid tokens before the chunk (and valid prefix tokens): block count.
  int cnt = 0;
  for (int t = threadIdx.x; t < t0; t += blockDim.x) cnt += tm[t] != 0;
  if (pmask) {
    const uint8_t* pm = pmask + (long long)b * pmask_bs;
    for (int t = threadIdx.x; t < P; t += blockDim.x) cnt += pm[t] != 0;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  if (lane == 0) s_count[warp] = cnt;
  __syncthreads();
  if (warp == 0) {
    int base = 0;
#pragma unroll
    for (int w = 0; w < kRopeThreads / 32; ++w) base += s_count[w];
    // inclusive scan of the chunk's own mask bits
    int v = (lane < nt && tm[t0 + lane] != 0) ? 1 : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += y;
    }
    if (lane < nt) {
      const int pos = base + v - 1;
      s_pos[lane] = pos;
      if (pos_out) pos_out[(long long)b * S + t0 + lane] = pos;
    }
  }
  __syncthreads();

  // cos / sin table for the chunk: angle = pos * base^(-2i/d), reduced in fp64.
  float* cs = tab;
  float* sn = tab + kRopeTokens * half;
  const double two_pi = 6.283185307179586476925286766559;
  for (int idx = threadIdx.x; idx < nt * half; idx += blockDim.x) {
    const int tl = idx / half, i = idx % half;
    const double inv = exp2(-2.0 * (double)i / (double)d * log2_base);
    double ang = (double)s_pos[tl] * inv;
    ang -= two_pi * rint(ang / two_pi);
    float sv, cv;
    sincosf((float)ang, &sv, &cv);
    cs[idx] = cv;
    sn[idx] = sv;
  }
  __syncthreads();
  rope_rows(q, Hq, d, S, b, t0, nt, cs, sn);
  if (k) rope_rows(k, Hkv, d, S, b, t0, nt, cs, sn);
}

template <typename T>
__global__ void __launch_bounds__(256)
    euler_kernel(float* __restrict__ x, const T* __restrict__ v, float dt, long long n) {
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

cudaError_t launch_rope(const RopeParams& p, cudaStream_t st) {
  dim3 grid((p.S + kRopeTokens - 1) / kRopeTokens, p.B);
  const size_t smem = (size_t)2 * kRopeTokens * (p.d / 2) * sizeof(float);
  const double log2_base = log2((double)p.base);
  if (p.f32) {
    rope_kernel<float><<<grid, kRopeThreads, smem, st>>>(
        static_cast<float*>(p.q), static_cast<float*>(p.k), p.tmask, p.tmask_bs, p.pmask,
        p.pmask_bs, p.S, p.P, p.Hq, p.Hkv, p.d, log2_base, p.pos_out);
  } else {
    rope_kernel<__nv_bfloat16><<<grid, kRopeThreads, smem, st>>>(
        static_cast<__nv_bfloat16*>(p.q), static_cast<__nv_bfloat16*>(p.k), p.tmask, p.tmask_bs,
        p.pmask, p.pmask_bs, p.S, p.P, p.Hq, p.Hkv, p.d, log2_base, p.pos_out);
  }
  return cudaGetLastError();
}

cudaError_t launch_euler(float* x, const void* v, bool v_f32, float dt, long long n,
                         cudaStream_t st) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long blocks_needed = (n / 4 + 255) / 256 + 1;
  const int grid = (int)std::min<long long>(blocks_needed, (long long)sms * 8);
  if (v_f32) {
    euler_kernel<float><<<grid, 256, 0, st>>>(x, static_cast<const float*>(v), dt, n);
  } else {
    euler_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(x, static_cast<const __nv_bfloat16*>(v),
                                                      dt, n);
  }
  return cudaGetLastError();
}

}  // namespace piattn

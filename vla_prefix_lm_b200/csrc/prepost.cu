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
// Both kernels are HBM-bound elementwise passes.  RoPE: a thread owns one
// (token, N-column slice of the first half) and the matching slice of the
// second half; it forms that slice's angles once (pos * base^(-2i/d), the
// inverse frequencies tabulated in fp64 per CTA and the product reduced modulo
// 2*pi in fp64, so that large positions keep fp32-level accuracy) and applies
// them to every head of q and k with 16-byte vector loads and stores.  The
// head loads are issued before the position prologue (a block count of the
// mask bytes before the CTA's tokens), so the prologue hides under their
// latency; tokens per CTA are chosen so that a CTA has 128 busy threads.
#include <cstdint>

#include "launch.h"

namespace piattn {

namespace {

constexpr int kRopeThreads = 128;
constexpr int kRopeMaxTok = 32;
constexpr int kRopeHeadBatch = 8;              // head vectors in flight per thread

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

// Row of head h (q heads first, then k heads) of token t.
template <typename T>
__device__ __forceinline__ T* head_row(T* q, T* k, int Hq, int Hkv, int d, long long bt, int h) {
  return h < Hq ? q + (bt * Hq + h) * d : k + (bt * Hkv + (h - Hq)) * d;
}

template <typename T>
__global__ void __launch_bounds__(kRopeThreads)
    rope_kernel(T* q, T* k, const uint8_t* tmask, long long tmask_bs, const uint8_t* pmask,
                long long pmask_bs, int S, int P, int Hq, int Hkv, int d, int tok_per_cta,
                double log2_base, int32_t* pos_out) {
  constexpr int N = Vec<T>::N;
  __shared__ double s_inv[128];                 // base^(-2i/d), i < d/2 <= 128
  __shared__ int s_count[kRopeThreads / 32];
  const int b = blockIdx.y;
  const int t0 = blockIdx.x * tok_per_cta;
  const int nt = min(tok_per_cta, S - t0);
  const int half = d / 2;
  const int vpr = half / N;                     // vectors per half row
  const int tl = threadIdx.x / vpr, vi = threadIdx.x % vpr;
  const bool active = tl < nt;
  const int Ht = Hq + (k ? Hkv : 0);
  const long long bt = (long long)b * S + t0 + tl;
  const uint8_t* tm = tmask + (long long)b * tmask_bs;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  uint4 ra[kRopeHeadBatch], rc[kRopeHeadBatch];
  auto load_batch = [&](int h0) {
#pragma unroll
    for (int j = 0; j < kRopeHeadBatch; ++j) {
      if (active && h0 + j < Ht) {
        const T* row = head_row(q, k, Hq, Hkv, d, bt, h0 + j);
        ra[j] = *reinterpret_cast<const uint4*>(row + vi * N);
        rc[j] = *reinterpret_cast<const uint4*>(row + half + vi * N);
      }
    }
  };
  load_batch(0);

  // Valid tokens before the CTA's first token (and valid prefix tokens).
  int cnt = 0;
  for (int t = threadIdx.x; t < t0; t += blockDim.x) cnt += tm[t] != 0;
  if (pmask) {
    const uint8_t* pm = pmask + (long long)b * pmask_bs;
    for (int t = threadIdx.x; t < P; t += blockDim.x) cnt += pm[t] != 0;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  if (lane == 0) s_count[warp] = cnt;
  for (int i = threadIdx.x; i < half; i += blockDim.x)
    s_inv[i] = exp2(-2.0 * (double)i / (double)d * log2_base);
  __syncthreads();
  if (!active) return;
  int pos = -1;
#pragma unroll
  for (int w = 0; w < kRopeThreads / 32; ++w) pos += s_count[w];
  for (int u = 0; u <= tl; ++u) pos += tm[t0 + u] != 0;
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

  for (int h0 = 0;;) {
#pragma unroll
    for (int j = 0; j < kRopeHeadBatch; ++j) {
      if (h0 + j < Ht) {
        float a[N], c[N], o1[N], o2[N];
        unpack(ra[j], a, (T*)nullptr);
        unpack(rc[j], c, (T*)nullptr);
#pragma unroll
        for (int e = 0; e < N; ++e) {
          o1[e] = a[e] * cs[e] - c[e] * sn[e];
          o2[e] = c[e] * cs[e] + a[e] * sn[e];
        }
        T* row = head_row(q, k, Hq, Hkv, d, bt, h0 + j);
        *reinterpret_cast<uint4*>(row + vi * N) = pack(o1, (T*)nullptr);
        *reinterpret_cast<uint4*>(row + half + vi * N) = pack(o2, (T*)nullptr);
      }
    }
    h0 += kRopeHeadBatch;
    if (h0 >= Ht) break;
    load_batch(h0);
  }
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
  const int vpr = p.d / 2 / (p.f32 ? Vec<float>::N : Vec<__nv_bfloat16>::N);
  const int tok = std::max(1, std::min(kRopeMaxTok, kRopeThreads / vpr));
  dim3 grid((p.S + tok - 1) / tok, p.B);
  const double log2_base = log2((double)p.base);
  if (p.f32) {
    rope_kernel<float><<<grid, kRopeThreads, 0, st>>>(
        static_cast<float*>(p.q), static_cast<float*>(p.k), p.tmask, p.tmask_bs, p.pmask,
        p.pmask_bs, p.S, p.P, p.Hq, p.Hkv, p.d, tok, log2_base, p.pos_out);
  } else {
    rope_kernel<__nv_bfloat16><<<grid, kRopeThreads, 0, st>>>(
        static_cast<__nv_bfloat16*>(p.q), static_cast<__nv_bfloat16*>(p.k), p.tmask, p.tmask_bs,
        p.pmask, p.pmask_bs, p.S, p.P, p.Hq, p.Hkv, p.d, tok, log2_base, p.pos_out);
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

// backward.cu -- gradient of the joint masked attention (dq, dk, dv) for the
// prefill, the pass the training step runs under gradient ("VLA 代码精读 -
// OpenPI & StarVLA", 1.5 Pi0.compute_loss).
//
// With P = softmax(scale * q k^T) over the visible keys and O = P v (the
// forward's out and its natural-log lse per row), for each query row i:
//     D_i = dO_i . O_i
//     p_ij = exp(scale * q_i . k_j - lse_i),   dp_ij = dO_i . v_j
//     ds_ij = p_ij * (dp_ij - D_i)
//     dq_i = scale * sum_j ds_ij k_j
//     dk_j = scale * sum_i ds_ij q_i,   dv_j = sum_i p_ij dO_i
// (the sums over i include every query head that reads key/value head g).
//
// Three deterministic SIMT passes, no atomics:
//   1. the packed mask code of every token (block scan of ar_mask);
//   2. one warp per (b, i, h) query row: D_i, then dq_i over the row's visible
//      keys -- a prefix [0, end_i) of the sequence, since the block index is
//      non-decreasing along the tokens (cumsum of a 0/1 mask);
//   3. one warp per (b, j, g) key row: dk_j and dv_j over the queries that
//      see key j, every head of the group.
// A warp lane holds the elements c = lane + 32 e of a head vector (coalesced
// 64- or 128-byte rows per e); dot products reduce with xor shuffles.  All
// arithmetic is fp32; the gradients are written in fp32.
#include <cstdint>

#include "launch.h"
#include "mask.cuh"

namespace piattn {

namespace {

constexpr int kBwdWarps = 8;                     // warps per CTA in passes 2 and 3
constexpr int kMaxE = 8;                         // d / 32 <= 8

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__device__ __forceinline__ void warp_sum2(float& a, float& b) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, off);
    b += __shfl_xor_sync(0xffffffffu, b, off);
  }
}

__global__ void __launch_bounds__(1024)
    bwd_codes_kernel(const uint8_t* ar, const int32_t* seg, long long mask_bs, int S,
                     uint32_t* codes) {
  __shared__ int scratch[33];
  const int b = blockIdx.x;
  build_codes<uint32_t>(ar + (long long)b * mask_bs, seg ? seg + (long long)b * mask_bs : nullptr,
                        S, codes + (long long)b * S, scratch);
}

template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32)
    bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const T* __restrict__ out, const float* __restrict__ lse,
                  const T* __restrict__ dout, const uint32_t* __restrict__ codes,
                  float* __restrict__ dq, float* __restrict__ Dws, int B, int S, int Hq, int Hkv,
                  int d, float scale) {
  const long long row = (long long)blockIdx.x * kBwdWarps + (threadIdx.x >> 5);
  if (row >= (long long)B * S * Hq) return;                // whole warp leaves together
  const int lane = threadIdx.x & 31;
  const int h = (int)(row % Hq);
  const long long bi = row / Hq;                           // b * S + i
  const int b = (int)(bi / S);
  const int g = h / (Hq / Hkv);
  const int E = d >> 5;
  const long long qo = row * d;                            // [B, S, Hq, d]
  const uint32_t cq = codes[bi];
  float* dq_row = dq + qo;
  if (is_pad(cq)) {
    for (int e = 0; e < E; ++e) dq_row[lane + 32 * e] = 0.f;
    if (lane == 0) Dws[row] = 0.f;
    return;
  }
  float qr[kMaxE], dor[kMaxE], acc[kMaxE];
  float Dp = 0.f;
#pragma unroll
  for (int e = 0; e < kMaxE; ++e) {
    qr[e] = dor[e] = acc[e] = 0.f;
    if (e < E) {
      const int c = lane + 32 * e;
      qr[e] = ld(q + qo + c);
      dor[e] = ld(dout + qo + c);
      Dp += dor[e] * ld(out + qo + c);
    }
  }
  const float D = warp_sum(Dp);
  if (lane == 0) Dws[row] = D;
  const float L = lse[row];
  const uint32_t* cb = codes + (long long)b * S;
  const long long kv0 = ((long long)b * S * Hkv + g) * d;  // key 0 of head g
  const long long kv_step = (long long)Hkv * d;
  for (int j = 0; j < S; ++j) {
    const uint32_t ck = cb[j];
    if ((ck >> 2) > (cq >> 2)) break;                      // past the visible prefix
    if (!visible(cq, ck)) continue;
    const long long ko = kv0 + j * kv_step;
    float kr[kMaxE];
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int e = 0; e < kMaxE; ++e) {
      kr[e] = 0.f;
      if (e < E) {
        const int c = lane + 32 * e;
        kr[e] = ld(k + ko + c);
        s += qr[e] * kr[e];
        dp += dor[e] * ld(v + ko + c);
      }
    }
    warp_sum2(s, dp);
    const float p = expf(scale * s - L);
    const float ds = p * (dp - D);
#pragma unroll
    for (int e = 0; e < kMaxE; ++e) acc[e] += ds * kr[e];
  }
#pragma unroll
  for (int e = 0; e < kMaxE; ++e)
    if (e < E) dq_row[lane + 32 * e] = scale * acc[e];
}

template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32)
    bwd_dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                    const float* __restrict__ lse, const T* __restrict__ dout,
                    const uint32_t* __restrict__ codes, const float* __restrict__ Dws,
                    float* __restrict__ dk, float* __restrict__ dv, int B, int S, int Hq, int Hkv,
                    int d, float scale) {
  const long long row = (long long)blockIdx.x * kBwdWarps + (threadIdx.x >> 5);
  if (row >= (long long)B * S * Hkv) return;               // whole warp leaves together
  const int lane = threadIdx.x & 31;
  const int g = (int)(row % Hkv);
  const long long bj = row / Hkv;                          // b * S + j
  const int b = (int)(bj / S);
  const int group = Hq / Hkv;
  const int E = d >> 5;
  const long long ko = row * d;                            // [B, S, Hkv, d]
  const uint32_t ck = codes[bj];
  float kr[kMaxE], vr[kMaxE], ak[kMaxE], av[kMaxE];
#pragma unroll
  for (int e = 0; e < kMaxE; ++e) {
    kr[e] = vr[e] = ak[e] = av[e] = 0.f;
    if (e < E) {
      kr[e] = ld(k + ko + lane + 32 * e);
      vr[e] = ld(v + ko + lane + 32 * e);
    }
  }
  const uint32_t* cb = codes + (long long)b * S;
  if (!is_pad(ck)) {
    for (int i = 0; i < S; ++i) {
      const uint32_t cq = cb[i];
      if (!visible(cq, ck)) continue;
      for (int hh = 0; hh < group; ++hh) {
        const int h = g * group + hh;
        const long long r = ((long long)b * S + i) * Hq + h;   // query row
        const long long qo = r * d;
        float qr[kMaxE], dor[kMaxE];
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < kMaxE; ++e) {
          qr[e] = dor[e] = 0.f;
          if (e < E) {
            const int c = lane + 32 * e;
            qr[e] = ld(q + qo + c);
            dor[e] = ld(dout + qo + c);
            s += qr[e] * kr[e];
            dp += dor[e] * vr[e];
          }
        }
        warp_sum2(s, dp);
        const float p = expf(scale * s - lse[r]);
        const float ds = p * (dp - Dws[r]);
#pragma unroll
        for (int e = 0; e < kMaxE; ++e) {
          av[e] += p * dor[e];
          ak[e] += ds * qr[e];
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < kMaxE; ++e) {
    if (e < E) {
      dk[ko + lane + 32 * e] = scale * ak[e];
      dv[ko + lane + 32 * e] = av[e];
    }
  }
}

template <typename T>
cudaError_t launch_bwd_typed(const BwdParams& p, cudaStream_t st) {
  bwd_codes_kernel<<<p.B, 1024, 0, st>>>(p.ar, p.seg, p.mask_bs, p.S, p.codes);
  const long long qrows = (long long)p.B * p.S * p.Hq;
  const long long krows = (long long)p.B * p.S * p.Hkv;
  bwd_dq_kernel<T><<<(unsigned)((qrows + kBwdWarps - 1) / kBwdWarps), kBwdWarps * 32, 0, st>>>(
      static_cast<const T*>(p.q), static_cast<const T*>(p.k), static_cast<const T*>(p.v),
      static_cast<const T*>(p.out), p.lse, static_cast<const T*>(p.dout), p.codes, p.dq, p.D, p.B,
      p.S, p.Hq, p.Hkv, p.d, p.scale);
  bwd_dkdv_kernel<T><<<(unsigned)((krows + kBwdWarps - 1) / kBwdWarps), kBwdWarps * 32, 0, st>>>(
      static_cast<const T*>(p.q), static_cast<const T*>(p.k), static_cast<const T*>(p.v), p.lse,
      static_cast<const T*>(p.dout), p.codes, p.D, p.dk, p.dv, p.B, p.S, p.Hq, p.Hkv, p.d,
      p.scale);
  return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(int B, int S, int Hq) {
  const size_t codes = ((size_t)B * S * sizeof(uint32_t) + 255) & ~(size_t)255;
  return codes + (size_t)B * S * Hq * sizeof(float);
}

cudaError_t launch_backward(const BwdParams& p, cudaStream_t st) {
  return p.f32 ? launch_bwd_typed<float>(p, st) : launch_bwd_typed<__nv_bfloat16>(p, st);
}

}  // namespace piattn

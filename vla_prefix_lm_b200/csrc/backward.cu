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

constexpr int kBwdWarps = 16;                    // rows (one per warp) a CTA owns
constexpr int kTile = 16;                        // rows of the other side staged at a time
constexpr int kMaxD = 256;
constexpr int kMaxE = kMaxD / 32;

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

// Loads the tile's rows into shared memory as fp32: row r of the tile is
// src + row_off(r) * d (a (token, head) row of [B, S, H, d]) or zeros when
// row_off(r) < 0.  Every thread of the CTA takes part.
template <typename T, typename RowOff>
__device__ __forceinline__ void stage_rows(float (*dst)[kMaxD], const T* __restrict__ src,
                                           int d, RowOff row_off) {
  for (int t = threadIdx.x; t < kTile * d; t += blockDim.x) {
    const int r = t / d, c = t - r * d;
    const long long o = row_off(r);
    dst[r][c] = o >= 0 ? ld(src + o * d + c) : 0.f;
  }
}

// dq: a CTA holds kBwdWarps query rows of one (batch element, key/value head
// g) -- the flattened (token, head of g's group) rows rho = token * group + hh
// -- one per warp, and streams the visible keys of head g through shared
// memory kTile at a time.
template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32)
    bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const T* __restrict__ out, const float* __restrict__ lse,
                  const T* __restrict__ dout, const uint32_t* __restrict__ codes,
                  float* __restrict__ dq, float* __restrict__ Dws, int S, int Hq, int Hkv, int d,
                  float scale) {
  __shared__ float ks[kTile][kMaxD];
  __shared__ float vs[kTile][kMaxD];
  __shared__ uint32_t cks[kTile];
  const int group = Hq / Hkv;
  const long long rows_g = (long long)S * group;           // rho range of one (b, g)
  const long long chunks = (rows_g + kBwdWarps - 1) / kBwdWarps;
  const long long bg = blockIdx.x / chunks;                // b * Hkv + g
  const long long rho0 = (blockIdx.x - bg * chunks) * kBwdWarps;
  const int b = (int)(bg / Hkv), g = (int)(bg - (long long)b * Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = d >> 5;
  const long long rho = rho0 + warp;
  const bool valid = rho < rows_g;
  const int i = valid ? (int)(rho / group) : 0;
  const int h = g * group + (valid ? (int)(rho - (long long)i * group) : 0);
  const long long row = ((long long)b * S + i) * Hq + h;
  const uint32_t* cb = codes + (long long)b * S;
  const uint32_t cq = valid ? cb[i] : 3u;                  // invalid rows act as padding
  const bool live = valid && !is_pad(cq);

  float qr[kMaxE], dor[kMaxE], acc[kMaxE];
  float Dp = 0.f;
#pragma unroll
  for (int e = 0; e < kMaxE; ++e) {
    qr[e] = dor[e] = acc[e] = 0.f;
    if (live && e < E) {
      const int c = lane + 32 * e;
      qr[e] = ld(q + row * d + c);
      dor[e] = ld(dout + row * d + c);
      Dp += dor[e] * ld(out + row * d + c);
    }
  }
  const float D = warp_sum(Dp);
  const float L = live ? lse[row] : 0.f;
  if (valid && lane == 0) Dws[row] = live ? D : 0.f;

  // Keys past the visible prefix of the chunk's last token are seen by no row.
  const long long rho_last = min(rho0 + kBwdWarps, rows_g) - 1;
  const uint32_t cs_max = cb[(int)(rho_last / group)] >> 2;
  for (int j0 = 0; j0 < S && (cb[j0] >> 2) <= cs_max; j0 += kTile) {
    __syncthreads();                                       // previous tile consumed
    auto key_off = [&](int r) -> long long {
      const int j = j0 + r;
      return j < S ? ((long long)b * S + j) * Hkv + g : -1;
    };
    stage_rows(ks, k, d, key_off);
    stage_rows(vs, v, d, key_off);
    if (threadIdx.x < kTile) cks[threadIdx.x] = j0 + (int)threadIdx.x < S ? cb[j0 + threadIdx.x] : 3u;
    __syncthreads();
    if (!live) continue;
    for (int jj = 0; jj < kTile; ++jj) {
      if (!visible(cq, cks[jj])) continue;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < kMaxE; ++e) {
        if (e < E) {
          s += qr[e] * ks[jj][lane + 32 * e];
          dp += dor[e] * vs[jj][lane + 32 * e];
        }
      }
      warp_sum2(s, dp);
      const float ds = expf(scale * s - L) * (dp - D);
#pragma unroll
      for (int e = 0; e < kMaxE; ++e)
        if (e < E) acc[e] += ds * ks[jj][lane + 32 * e];
    }
  }
  if (valid) {
#pragma unroll
    for (int e = 0; e < kMaxE; ++e)
      if (e < E) dq[row * d + lane + 32 * e] = scale * acc[e];
  }
}

// dk, dv: a CTA holds kBwdWarps consecutive keys of one (batch element, head
// g), one per warp, and streams the query rows of g's group -- flattened
// (token, head) rows rho = token * group + hh with their q, dO, lse and D --
// through shared memory kTile rows at a time, skipping tiles whose last token
// has a smaller block index than the CTA's first key (no row there sees any
// of its keys).
template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32)
    bwd_dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                    const float* __restrict__ lse, const T* __restrict__ dout,
                    const uint32_t* __restrict__ codes, const float* __restrict__ Dws,
                    float* __restrict__ dk, float* __restrict__ dv, int S, int Hq, int Hkv, int d,
                    float scale) {
  __shared__ float qs[kTile][kMaxD];
  __shared__ float dos[kTile][kMaxD];
  __shared__ float Ls[kTile], Ds[kTile];
  __shared__ uint32_t cqs[kTile];
  const int group = Hq / Hkv;
  const int chunks = (S + kBwdWarps - 1) / kBwdWarps;
  const long long bg = blockIdx.x / chunks;                // b * Hkv + g
  const int j0 = (int)(blockIdx.x - bg * chunks) * kBwdWarps;
  const int b = (int)(bg / Hkv), g = (int)(bg - (long long)b * Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = d >> 5;
  const int j = j0 + warp;
  const bool valid = j < S;
  const long long krow = ((long long)b * S + (valid ? j : 0)) * Hkv + g;
  const uint32_t* cb = codes + (long long)b * S;
  const uint32_t ck = valid ? cb[j] : 3u;
  const bool live = valid && !is_pad(ck);
  float kr[kMaxE], vr[kMaxE], ak[kMaxE], av[kMaxE];
#pragma unroll
  for (int e = 0; e < kMaxE; ++e) {
    kr[e] = vr[e] = ak[e] = av[e] = 0.f;
    if (live && e < E) {
      kr[e] = ld(k + krow * d + lane + 32 * e);
      vr[e] = ld(v + krow * d + lane + 32 * e);
    }
  }
  const uint32_t cs_min = cb[j0] >> 2;                     // smallest block index of the keys
  const long long rows_g = (long long)S * group;
  for (long long r0 = 0; r0 < rows_g; r0 += kTile) {
    const int t_last = (int)(min(r0 + kTile, rows_g) - 1) / group;
    if ((cb[t_last] >> 2) < cs_min) continue;             // uniform: no row sees these keys
    __syncthreads();                                       // previous tile consumed
    auto q_off = [&](int r) -> long long {
      const long long rho = r0 + r;
      if (rho >= rows_g) return -1;
      const int t = (int)(rho / group);
      return ((long long)b * S + t) * Hq + g * group + (int)(rho - (long long)t * group);
    };
    stage_rows(qs, q, d, q_off);
    stage_rows(dos, dout, d, q_off);
    if (threadIdx.x < kTile) {
      const long long o = q_off((int)threadIdx.x);
      const int t = (int)((r0 + threadIdx.x) / group);
      cqs[threadIdx.x] = o >= 0 ? cb[t] : 3u;
      Ls[threadIdx.x] = o >= 0 ? lse[o] : 0.f;
      Ds[threadIdx.x] = o >= 0 ? Dws[o] : 0.f;
    }
    __syncthreads();
    if (!live) continue;
    for (int rr = 0; rr < kTile; ++rr) {
      if (!visible(cqs[rr], ck)) continue;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < kMaxE; ++e) {
        if (e < E) {
          s += qs[rr][lane + 32 * e] * kr[e];
          dp += dos[rr][lane + 32 * e] * vr[e];
        }
      }
      warp_sum2(s, dp);
      const float p = expf(scale * s - Ls[rr]);
      const float ds = p * (dp - Ds[rr]);
#pragma unroll
      for (int e = 0; e < kMaxE; ++e) {
        if (e < E) {
          av[e] += p * dos[rr][lane + 32 * e];
          ak[e] += ds * qs[rr][lane + 32 * e];
        }
      }
    }
  }
  if (valid) {
#pragma unroll
    for (int e = 0; e < kMaxE; ++e) {
      if (e < E) {
        dk[krow * d + lane + 32 * e] = scale * ak[e];
        dv[krow * d + lane + 32 * e] = av[e];
      }
    }
  }
}

template <typename T>
cudaError_t launch_bwd_typed(const BwdParams& p, cudaStream_t st) {
  bwd_codes_kernel<<<p.B, 1024, 0, st>>>(p.ar, p.seg, p.mask_bs, p.S, p.codes);
  const long long group = p.Hq / p.Hkv;
  const long long dq_blocks = (long long)p.B * p.Hkv * ((p.S * group + kBwdWarps - 1) / kBwdWarps);
  const long long dk_blocks = (long long)p.B * p.Hkv * ((p.S + kBwdWarps - 1) / kBwdWarps);
  bwd_dq_kernel<T><<<(unsigned)dq_blocks, kBwdWarps * 32, 0, st>>>(
      static_cast<const T*>(p.q), static_cast<const T*>(p.k), static_cast<const T*>(p.v),
      static_cast<const T*>(p.out), p.lse, static_cast<const T*>(p.dout), p.codes, p.dq, p.D, p.S,
      p.Hq, p.Hkv, p.d, p.scale);
  bwd_dkdv_kernel<T><<<(unsigned)dk_blocks, kBwdWarps * 32, 0, st>>>(
      static_cast<const T*>(p.q), static_cast<const T*>(p.k), static_cast<const T*>(p.v), p.lse,
      static_cast<const T*>(p.dout), p.codes, p.D, p.dk, p.dv, p.S, p.Hq, p.Hkv, p.d, p.scale);
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

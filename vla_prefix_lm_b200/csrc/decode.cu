// decode.cu -- the suffix pass when the suffix has few query rows (Sq * Hq <=
// 8), such as Pi0-FAST's token-by-token decode against its KV cache
// ("Pi0-FAST 模型架构", 4.1 KV 缓存推理: each new token attends to the cached
// keys and values plus itself).
//
// With eight or fewer query rows the work is reading the cache: every cached
// key and value row (512 bytes each) feeds at most eight dot products of
// length 256, and a 256-row tcgen05 tile would be 97 % empty.  The kernel
// spreads the cache over the whole GPU and keeps the arithmetic off the
// critical path with warp-level tensor-core instructions:
//
//  * one cluster of 8 CTAs per batch element; the element's keys form 16-key
//    tiles (its cache, then one tile of suffix keys) that the 8 CTAs share
//    out in contiguous runs, each CTA bringing its tiles by TMA into a
//    four-stage ring of 128-byte-swizzled K and V tiles in shared memory;
//  * warp w takes every fourth tile through stage w (so each stage is
//    refilled as soon as its one reader is done): the scores transposed, S^T = K Q^T with mma.m16n8k16, so that the 8 query
//    rows fill the n8 side and no MMA row is padding (K fragments by
//    ldmatrix, Q^T held in registers); an online softmax per query column in
//    fp32; then O^T += V^T P^T with mma.m16n8k16, V^T fragments from
//    ldmatrix.trans and P^T from the score accumulator by an in-register
//    8x8 transpose (movmatrix);
//  * the 4 warp partials (m, l, O) merge in shared memory; each CTA then
//    pushes column block k of its merged rows into CTA k's shared memory
//    (distributed shared-memory stores, one cluster barrier), and CTA k
//    finishes those 32 of the 256 output columns (the log-sum-exp rule).
// Every cache byte is read from HBM once; no workspace, no second launch.
// The mask is the prefix-LM rule: cached keys are visible to every valid
// query row (and hidden where the cache validity mask says so), suffix keys
// by the block-index rule over the suffix tokens (mask.cuh).  The TMA waits
// are bounded; a timeout leaves the output unwritten and is reported in the
// status word.
#include <cfloat>

#include "launch.h"
#include "mask.cuh"

namespace piattn {

namespace {

constexpr int kDecThreads = 128;          // 4 warps
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecCluster = 8;            // CTAs per batch element
constexpr int kDecRows = 8;               // query rows (Sq * Hq) at most
constexpr int kDecD = 256;
constexpr int kDecTile = kDecodeTileKeys; // keys per TMA tile (one warp's m16 tile)
constexpr int kTileBytes = kDecTile * kDecD * 2;    // 8 KB: 4 blocks of [16 x 128 B]
constexpr int kStages = kDecWarps;        // one stage per warp
constexpr int kPartStride = kDecD + 4;    // fp32 partial rows: 4-bank skew, conflict-free

struct DecSmem {
  float m[kDecWarps][kDecRows];
  float l[kDecWarps][kDecRows];
  uint32_t codes[kDecRows];               // suffix tokens' packed codes
  // What the 8 CTAs of the cluster push to this one: their merged partials
  // for this CTA's 32 output columns, and their (m, l) per row.
  float o_in[kDecCluster][kDecRows][32];
  float2 ml_in[kDecCluster][kDecRows];
  uint64_t full[kStages];
  int timed_out;
  int peer_timed_out;                     // set by a CTA of the cluster that timed out
};
// The ring (K, V per stage) comes first; after the loop its first 33 KB hold
// the warp partials O[warp][row][kPartStride] (fp32), then the CTA's.
constexpr int kRingBytes = kStages * 2 * kTileBytes;              // 64 KB
constexpr int kDecSmemBytes = kRingBytes + (int)sizeof(DecSmem) + 1024;
static_assert(kDecWarps * kDecRows * kPartStride * 4 <= kRingBytes, "partials do not fit the ring");

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared-memory byte offset of the 16-byte chunk holding columns [d, d + 8) of
// row j in a [16 x 256] bf16 tile loaded by one TMA box (64, 16, 4, 1) with
// the 128-byte swizzle: four [16 x 64] blocks, chunk c of row j at c ^ (j % 8).
__device__ __forceinline__ uint32_t chunk_off(int j, int d) {
  return (uint32_t)((d >> 6) * (kDecTile * 128) + j * 128 + ((((d & 63) >> 3) ^ (j & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D (16x8 fp32) += A (16x16 bf16) * B (16x8 bf16).
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 bf16 matrix held one row pair per lane (lane (g, t4):
// row g, columns 2 t4, 2 t4 + 1).
__device__ __forceinline__ uint32_t movm_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ void st_cluster_f32x2(uint32_t addr, float2 v) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(v.x), "f"(v.y)
               : "memory");
}

__global__ void __cluster_dims__(kDecCluster, 1, 1) __launch_bounds__(kDecThreads)
    decode_kernel(const __grid_constant__ DecodeParams p, const DevCtl ctl) {
  extern __shared__ __align__(1024) uint8_t dec_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dec_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  DecSmem& sm = *reinterpret_cast<DecSmem*>(ring + kRingBytes);
  float* opart = reinterpret_cast<float*>(ring);     // [warp][row][kPartStride] after the loop

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int g = lane >> 2, t4 = lane & 3;             // mma fragment coordinates
  const uint32_t crank = cluster_ctarank();
  const int b = blockIdx.y;
  const int R = p.Sq * p.Hq;

  // Units of the batch element: its 16-key cache tiles, then one tile of
  // suffix keys; CTA c of the cluster takes units [U c / 8, U (c + 1) / 8), so
  // the suffix tile (the last unit) falls to the last CTA and no CTA has more
  // than one tile above another.
  const int n_ct = (p.P + kDecTile - 1) / kDecTile;
  const int n_units = n_ct + 1;
  const int u0 = n_units * (int)crank / kDecCluster;
  const int u1 = n_units * ((int)crank + 1) / kDecCluster;
  const int n_tiles = u1 - u0;

  auto issue = [&](int i) {            // one thread: TMA of tile i into stage i % 4
    const int s = i % kStages;
    const int u = u0 + i;
    uint8_t* kt = ring + s * 2 * kTileBytes;
    mbar_arrive_expect_tx(&sm.full[s], 2 * kTileBytes);
    if (u < n_ct) {
      tma_load_4d(kt, &p.map_kc, &sm.full[s], 0, u * kDecTile, 0, b);
      tma_load_4d(kt + kTileBytes, &p.map_vc, &sm.full[s], 0, u * kDecTile, 0, b);
    } else {
      tma_load_4d(kt, &p.map_k, &sm.full[s], 0, 0, 0, b);
      tma_load_4d(kt + kTileBytes, &p.map_v, &sm.full[s], 0, 0, 0, b);
    }
  };
  // Nothing above touched global memory: it may overlap the previous kernel
  // in the stream, whose results are visible from here on.
  pdl_wait();
  pdl_launch_dependents();
  if (t == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[s], 1);
    sm.timed_out = 0;
    sm.peer_timed_out = 0;
    fence_barrier_init();
    for (int i = 0; i < kStages && i < n_tiles; ++i) issue(i);
    const uint8_t* ar = p.ar + (long long)b * p.mask_bs;
    const int32_t* seg = p.seg ? p.seg + (long long)b * p.mask_bs : nullptr;
    uint32_t cs = 0;
    for (int s = 0; s < kDecRows; ++s) {
      if (s < p.Sq) {
        cs += ar[s] != 0 ? 1u : 0u;
        sm.codes[s] = make_code(cs, seg ? seg[s] : 0);
      } else {
        sm.codes[s] = 3u;        // no such token: acts as padding
      }
    }
  }
  __syncthreads();
  // Every CTA of the cluster is running from here on (its partials are pushed
  // into the others' shared memory after the loop).
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  // The scores are computed transposed, S^T [16 keys x 8 query rows] = K Q^T,
  // so that the 8 query rows fill the n8 side of m16n8k16 and no MMA row is
  // padding.  Q^T is the B operand, read straight from global memory into
  // registers: lane (g, t4) holds Q[g][16 kk + 2 t4, + 1] and
  // Q[g][16 kk + 2 t4 + 8, + 9] (rows past R are zeros).
  uint32_t qb[16][2];
  {
    const uint32_t* qg = reinterpret_cast<const uint32_t*>(p.q + ((long long)b * R + g) * kDecD);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      qb[kk][0] = g < R ? qg[8 * kk + t4] : 0u;
      qb[kk][1] = g < R ? qg[8 * kk + 4 + t4] : 0u;
    }
  }
  // This lane's two query rows (score columns) 2 t4 and 2 t4 + 1.
  const int qr0 = 2 * t4, qr1 = 2 * t4 + 1;
  const uint32_t code0 = sm.codes[min(qr0 / p.Hq, kDecRows - 1)];
  const uint32_t code1 = sm.codes[min(qr1 / p.Hq, kDecRows - 1)];
  const bool row0_ok = qr0 < R && !is_pad(code0);
  const bool row1_ok = qr1 < R && !is_pad(code1);
  const float sl2 = p.scale_log2;

  // Warp w takes the tiles i = w, w + 4, ... through stage w, all 16 keys of
  // each.  O^T [256 x 8 rows] accumulates 16 column blocks of m16n8k16.
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  bool ok = true;

  for (int i = warp; i < n_tiles; i += kStages) {
    const int s = warp;
    // A timed-out wait skips the work; the others stop at their next tile.
    const bool landed = ok && mbar_wait(&sm.full[s], (i / kStages) & 1, ctl);
    if (ok && !landed) sm.timed_out = 1;
    if (landed) {
      const int u = u0 + i;
      const bool suf = u >= n_ct;
      const int kbase = suf ? 0 : u * kDecTile;               // key index of tile row 0
      const int n_here = suf ? p.Sq : min(kDecTile, p.P - kbase);
      const uint32_t kt = smem_u32(ring + s * 2 * kTileBytes);
      const uint32_t vt = kt + kTileBytes;
      const int j0 = 0;                                        // the warp's tile rows

      // S^T = K Q^T over 16 k-steps, two accumulation chains.  A fragments of
      // K rows j0 .. j0 + 15: matrix m of an x4 load holds rows 8 (m & 1) ..,
      // columns 8 (m >> 1) .. of the k-step.
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
      const int krow = j0 + 8 * ((lane >> 3) & 1) + (lane & 7);
#pragma unroll
      for (int kk = 0; kk < 16; kk += 2) {
        uint32_t a0, a1, a2, a3, e0, e1, e2, e3;
        ldsm_x4(kt + chunk_off(krow, 16 * kk + 8 * (lane >> 4)), a0, a1, a2, a3);
        ldsm_x4(kt + chunk_off(krow, 16 * kk + 16 + 8 * (lane >> 4)), e0, e1, e2, e3);
        mma16816(sa, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
        mma16816(sb, e0, e1, e2, e3, qb[kk + 1][0], qb[kk + 1][1]);
      }
      // sc[0]: key j0 + g, row qr0; [1]: j0 + g, qr1; [2]: j0 + g + 8, qr0; [3]: j0 + g + 8, qr1
      float sc[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[e] = (sa[e] + sb[e]) * sl2;
      {
        const int ja = j0 + g, jb = ja + 8;
        bool va0, va1, vb0, vb1;
        if (suf) {
          const uint32_t ca = sm.codes[min(ja, kDecRows - 1)], cb = sm.codes[min(jb, kDecRows - 1)];
          va0 = ja < n_here && visible(code0, ca);
          va1 = ja < n_here && visible(code1, ca);
          vb0 = jb < n_here && visible(code0, cb);
          vb1 = jb < n_here && visible(code1, cb);
        } else {
          bool ka = ja < n_here, kb = jb < n_here;
          if (p.cache_valid) {
            const uint8_t* cv = p.cache_valid + (long long)b * p.P + kbase;
            ka = ka && cv[ja] != 0;
            kb = kb && cv[jb] != 0;
          }
          va0 = ka && row0_ok;
          va1 = ka && row1_ok;
          vb0 = kb && row0_ok;
          vb1 = kb && row1_ok;
        }
        sc[0] = va0 ? sc[0] : -INFINITY;
        sc[1] = va1 ? sc[1] : -INFINITY;
        sc[2] = vb0 ? sc[2] : -INFINITY;
        sc[3] = vb1 ? sc[3] : -INFINITY;
      }
      // Column maxima over the 16 keys: the 8 lanes of equal t4.
      float x0 = fmaxf(sc[0], sc[2]), x1 = fmaxf(sc[1], sc[3]);
#pragma unroll
      for (int sh = 4; sh <= 16; sh <<= 1) {
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, sh));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, sh));
      }
      // Lazy rescaling: O and l change reference only when a row's maximum
      // grows by more than 8 (log2 units), so p stays <= 256.
      if (x0 > m0 + 8.f) {
        const float alpha = m0 == -INFINITY ? 0.f : ex2f(m0 - x0);
        l0 *= alpha;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          o[n][0] *= alpha;
          o[n][2] *= alpha;
        }
        m0 = x0;
      }
      if (x1 > m1 + 8.f) {
        const float alpha = m1 == -INFINITY ? 0.f : ex2f(m1 - x1);
        l1 *= alpha;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          o[n][1] *= alpha;
          o[n][3] *= alpha;
        }
        m1 = x1;
      }
      const float pa0 = m0 == -INFINITY ? 0.f : ex2f(sc[0] - m0);
      const float pa1 = m1 == -INFINITY ? 0.f : ex2f(sc[1] - m1);
      const float pb0 = m0 == -INFINITY ? 0.f : ex2f(sc[2] - m0);
      const float pb1 = m1 == -INFINITY ? 0.f : ex2f(sc[3] - m1);
      l0 += pa0 + pb0;
      l1 += pa1 + pb1;
      // P^T as the B operand of O^T += V^T P^T: lane (g, t4) needs
      // P[row g][keys 2 t4, 2 t4 + 1] (and + 8); it holds P[keys g, g + 8][rows
      // 2 t4, 2 t4 + 1], so each 8x8 block is transposed in registers.
      const uint32_t pb_lo = movm_trans(cvt_bf16x2(pa0, pa1));
      const uint32_t pb_hi = movm_trans(cvt_bf16x2(pb0, pb1));
      // A fragments of V^T (rows d, columns keys) from V rows j0 .. j0 + 15 by
      // transposing loads: matrix m holds keys 8 (m >> 1) .., columns 8 (m & 1) ..
      const int vrow = j0 + 8 * (lane >> 4) + (lane & 7);
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        uint32_t v0, v1, v2, v3;
        ldsm_x4_t(vt + chunk_off(vrow, 16 * n + 8 * ((lane >> 3) & 1)), v0, v1, v2, v3);
        mma16816(o[n], v0, v1, v2, v3, pb_lo, pb_hi);
      }
    }
    __syncwarp();                            // the warp is done with stage s
    ok = *reinterpret_cast<volatile int*>(&sm.timed_out) == 0;
    if (ok && lane == 0 && i + kStages < n_tiles) issue(i + kStages);
  }
  __syncthreads();
  ok = sm.timed_out == 0;
  if (!ok) {
    // Leave without writing (the status word holds PI_ERR_TIMEOUT), after a
    // bounded wait for the copies issued, and after the cluster's barriers.
    if (t == 0)
      for (int i = max(n_tiles - kStages, 0); i < n_tiles; ++i)
        (void)mbar_wait(&sm.full[i % kStages], (i / kStages) & 1, ctl);
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (t == 0)     // the others leave their columns unwritten too
      for (int k = 0; k < kDecCluster; ++k)
        asm volatile("st.shared::cluster.u32 [%0], 1;" ::"r"(
                         mapa_shared(smem_u32(&sm.peer_timed_out), (uint32_t)k))
                     : "memory");
    cluster_sync();
    return;
  }

  // ---------------------------------------- warp partials -> CTA partial
  // Row sums over the 8 lanes of equal t4.
#pragma unroll
  for (int sh = 4; sh <= 16; sh <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, sh);
    l1 += __shfl_xor_sync(0xffffffffu, l1, sh);
  }
  // o[n][0]: column 16 n + g, row qr0; [1]: 16 n + g, qr1; [2], [3]: column + 8.
  {
    float* ow = opart + warp * kDecRows * kPartStride;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      ow[qr0 * kPartStride + 16 * n + g] = o[n][0];
      ow[qr1 * kPartStride + 16 * n + g] = o[n][1];
      ow[qr0 * kPartStride + 16 * n + g + 8] = o[n][2];
      ow[qr1 * kPartStride + 16 * n + g + 8] = o[n][3];
    }
  }
  if (g == 0) {
    sm.m[warp][qr0] = m0;
    sm.m[warp][qr1] = m1;
    sm.l[warp][qr0] = l0;
    sm.l[warp][qr1] = l1;
  }
  __syncthreads();
  // thread t: row r = t / 16, columns 2 (t % 16) + 32 k (k < 8); column block
  // k of the merged row is pushed to CTA k of the cluster.
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  {
    const int r = t >> 4, dl = 2 * (t & 15);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm.m[w][r]);
    float f[kDecWarps], L = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      f[w] = M == -INFINITY ? 0.f : ex2f(sm.m[w][r] - M);
      L += f[w] * sm.l[w][r];
    }
    const uint32_t o_dst = smem_u32(&sm.o_in[crank][r][dl]);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float2 x = make_float2(0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float2 v = *reinterpret_cast<const float2*>(
            &opart[(w * kDecRows + r) * kPartStride + dl + 32 * k]);
        x.x += f[w] * v.x;
        x.y += f[w] * v.y;
      }
      st_cluster_f32x2(mapa_shared(o_dst, (uint32_t)k), x);
    }
    if ((t & 15) == 0) {
      const uint32_t ml_dst = smem_u32(&sm.ml_in[crank][r]);
#pragma unroll
      for (int k = 0; k < kDecCluster; ++k)
        st_cluster_f32x2(mapa_shared(ml_dst, (uint32_t)k), make_float2(M, L));
    }
  }
  // The pushes are visible to their owners, and all 8 CTAs' pushes to this
  // one have landed; nobody touches another CTA's shared memory after this.
  cluster_sync();
  // --------------------------------- CTA partials -> output (this CTA's columns)
  {
    const int r = t >> 4;                     // 8 rows x 16 threads
    const int dc = 2 * (t & 15);
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kDecCluster; ++c) M = fmaxf(M, sm.ml_in[c][r].x);
    float L = 0.f, x0 = 0.f, x1 = 0.f;
#pragma unroll
    for (int c = 0; c < kDecCluster; ++c) {
      const float2 ml = sm.ml_in[c][r];
      const float2 v = *reinterpret_cast<const float2*>(&sm.o_in[c][r][dc]);
      const float f = M == -INFINITY ? 0.f : ex2f(ml.x - M);
      L += f * ml.y;
      x0 += f * v.x;
      x1 += f * v.y;
    }
    if (r < R && sm.peer_timed_out == 0) {
      const float inv = L > 0.f ? 1.f / L : 0.f;   // a row that saw nothing writes 0
      *reinterpret_cast<__nv_bfloat162*>(p.out + ((long long)b * R + r) * kDecD +
                                          32 * (int)crank + dc) =
          __floats2bfloat162_rn(x0 * inv, x1 * inv);
    }
  }
}

}  // namespace

bool decode_applies(int Sq, int Hq) { return Sq >= 1 && Sq * Hq <= kDecRows; }

cudaError_t launch_decode(const DecodeParams& p, const DevCtl& ctl, cudaStream_t st) {
  // Per call: the attribute belongs to the device (and to the module, which a
  // device reset reloads).
  const cudaError_t attr = cudaFuncSetAttribute(
      decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmemBytes);
  if (attr != cudaSuccess) return attr;
  dim3 grid(kDecCluster, (unsigned)p.B);
  return launch_pdl(decode_kernel, grid, dim3(kDecThreads), kDecSmemBytes, st, p, ctl);
}

}  // namespace piattn

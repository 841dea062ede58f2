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
//  * one cluster of 8 CTAs per batch element; CTA q takes an eighth of the
//    cached keys (and the last CTA with keys also the suffix keys), in tiles
//    of 32 keys that TMA brings into a two-stage ring of 128-byte-swizzled
//    K and V tiles in shared memory;
//  * each of the 4 warps takes 8 keys of a tile: S = Q K^T with
//    mma.m16n8k16 (the 8 query rows padded to 16; Q fragments held in
//    registers, K fragments by ldmatrix), an online softmax of the 8 scores
//    per row in fp32 (two shuffles per maximum), then O += P V with
//    mma.m16n8k8, whose A operand is the score accumulator itself, converted
//    to bf16, and whose V fragments come from ldmatrix.trans;
//  * the 4 warp partials (m, l, O) merge in shared memory, then the 8 CTA
//    partials of the cluster through distributed shared memory, each CTA
//    finishing 32 of the 256 output columns (the log-sum-exp rule).
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
constexpr int kDecTile = 32;              // keys per TMA tile (8 per warp)
constexpr int kTileBytes = kDecTile * kDecD * 2;    // 16 KB: 4 blocks of [32 x 128 B]
constexpr int kStages = 2;

struct DecSmem {
  uint4 q[kDecRows * kDecD / 8];          // query rows, 16-byte chunk c of row r at c ^ r
  float m[kDecWarps][kDecRows];
  float l[kDecWarps][kDecRows];
  uint32_t codes[kDecRows];               // suffix tokens' packed codes
  uint64_t full[kStages];
  int timed_out;
};
// The ring (K, V per stage) comes first; after the loop its first 32 KB hold
// the warp partials O[warp][row][256] (fp32), then the CTA's.
constexpr int kRingBytes = kStages * 2 * kTileBytes;              // 64 KB
constexpr int kDecSmemBytes = kRingBytes + (int)sizeof(DecSmem) + 1024;
static_assert(kDecWarps * kDecRows * kDecD * 4 <= kRingBytes, "partials do not fit the ring");

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Shared-memory byte offset of the 16-byte chunk holding columns [d, d + 8) of
// row j in a [32 x 256] bf16 tile loaded by one TMA box (64, 32, 4, 1) with
// the 128-byte swizzle: four [32 x 64] blocks, chunk c of row j at c ^ (j % 8).
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

// D (16x8 fp32) += A (16x16 bf16, rows 8..15 zero) * B (16x8 bf16).
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// D (16x8 fp32) += A (16x8 bf16, rows 8..15 zero) * B (8x8 bf16).
__device__ __forceinline__ void mma1688(float (&c)[4], uint32_t a0, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(b0));
}

__global__ void __cluster_dims__(kDecCluster, 1, 1) __launch_bounds__(kDecThreads)
    decode_kernel(const __grid_constant__ DecodeParams p, const DevCtl ctl) {
  extern __shared__ __align__(1024) uint8_t dec_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dec_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  DecSmem& sm = *reinterpret_cast<DecSmem*>(ring + kRingBytes);
  float* opart = reinterpret_cast<float*>(ring);     // [warp][row][256] after the loop

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int g = lane >> 2, t4 = lane & 3;             // mma fragment coordinates
  const uint32_t crank = cluster_ctarank();
  const int b = blockIdx.y;
  const int R = p.Sq * p.Hq;

  // This CTA's tiles: 32-key tiles of its eighth of the cache, then (the last
  // CTA that has keys) one tile of suffix keys.
  const int c0 = (int)((long long)p.P * crank / kDecCluster);
  const int c1 = (int)((long long)p.P * (crank + 1) / kDecCluster);
  const int n_cache_tiles = (c1 - c0 + kDecTile - 1) / kDecTile;
  const bool has_suffix = crank == kDecCluster - 1;
  const int n_tiles = n_cache_tiles + (has_suffix ? 1 : 0);

  auto issue = [&](int i) {            // thread 0: TMA of tile i into stage i % 2
    const int s = i % kStages;
    uint8_t* kt = ring + s * 2 * kTileBytes;
    mbar_arrive_expect_tx(&sm.full[s], 2 * kTileBytes);
    if (i < n_cache_tiles) {
      tma_load_4d(kt, &p.map_kc, &sm.full[s], 0, c0 + i * kDecTile, 0, b);
      tma_load_4d(kt + kTileBytes, &p.map_vc, &sm.full[s], 0, c0 + i * kDecTile, 0, b);
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
  // The query rows through shared memory: coalesced 16-byte loads, rows past
  // R as zeros.
  {
    const uint4* qg = reinterpret_cast<const uint4*>(p.q + (long long)b * R * kDecD);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int c = t + kDecThreads * k;          // chunk index, 32 per row
      const int r = c >> 5, cc = c & 31;
      sm.q[r * 32 + (cc ^ r)] = r < R ? qg[c] : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __syncthreads();
  // Q fragments (rows 0..7 of the m16 tile; rows 8..15 are zero): lane (g, t4)
  // holds Q[g][16 kk + 2 t4, + 1] and Q[g][16 kk + 2 t4 + 8, + 9]; an x4 load
  // brings columns 32 h .. 32 h + 31 (k-steps 2 h and 2 h + 1).
  uint32_t qa[16][2];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    const int r = lane & 7, cc = 4 * h + (lane >> 3);
    ldsm_x4(smem_u32(&sm.q[r * 32 + (cc ^ r)]), qa[2 * h][0], qa[2 * h][1], qa[2 * h + 1][0],
            qa[2 * h + 1][1]);
  }
  const uint32_t my_code = sm.codes[min(g / p.Hq, kDecRows - 1)];
  const bool row_ok = g < R && !is_pad(my_code);
  const float sl2 = p.scale_log2;

  float o[32][4];
#pragma unroll
  for (int n = 0; n < 32; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run = -INFINITY, l_part = 0.f;
  bool ok = true;

  for (int i = 0; i < n_tiles; ++i) {
    const int s = i % kStages;
    // A timed-out wait skips the work but not the barrier at the end of the
    // iteration, so every thread passes the same barriers.
    if (ok && !mbar_wait(&sm.full[s], (i / kStages) & 1, ctl)) sm.timed_out = 1;
    if (!ok) {
      __syncthreads();
      continue;
    }
    const bool suf = i >= n_cache_tiles;
    const int kbase = suf ? 0 : c0 + i * kDecTile;           // key index of tile row 0
    const int n_here = suf ? p.Sq : min(kDecTile, c1 - kbase);
    const uint32_t kt = smem_u32(ring + s * 2 * kTileBytes);
    const uint32_t vt = kt + kTileBytes;
    const int j0 = 8 * warp;                                   // this warp's tile rows

    // S[16 x 8] = Q[16 x 256] K^T: x4 loads bring K rows j0..j0+7, columns 32 h..32 h+31
    // two independent accumulation chains (even and odd k-steps), summed at the end
    float sc[4] = {0.f, 0.f, 0.f, 0.f}, sd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      uint32_t k0, k1, k2, k3;
      ldsm_x4(kt + chunk_off(j0 + (lane & 7), 32 * h + 8 * (lane >> 3)), k0, k1, k2, k3);
      mma16816(sc, qa[2 * h][0], qa[2 * h][1], k0, k1);
      mma16816(sd, qa[2 * h + 1][0], qa[2 * h + 1][1], k2, k3);
    }
    // this lane's two scores: row g, tile rows j0 + 2 t4 and j0 + 2 t4 + 1
    float s0 = (sc[0] + sd[0]) * sl2, s1 = (sc[1] + sd[1]) * sl2;
    {
      const int ja = j0 + 2 * t4, jb = ja + 1;
      bool va = row_ok && ja < n_here, vb = row_ok && jb < n_here;
      if (suf) {
        va = va && visible(my_code, sm.codes[ja]);
        vb = vb && visible(my_code, sm.codes[jb]);
      } else if (p.cache_valid) {
        const uint8_t* cv = p.cache_valid + (long long)b * p.P + kbase;
        va = va && cv[ja] != 0;
        vb = vb && cv[jb] != 0;
      }
      s0 = va ? s0 : -INFINITY;
      s1 = vb ? s1 : -INFINITY;
    }
    float mx = fmaxf(s0, s1);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    // Lazy rescaling: O and l change reference only when the maximum grows by
    // more than 8 (log2 units), so p stays <= 256.
    if (mx > m_run + 8.f) {
      const float alpha = m_run == -INFINITY ? 0.f : ex2f(m_run - mx);
      l_part *= alpha;
#pragma unroll
      for (int n = 0; n < 32; ++n) {
        o[n][0] *= alpha;
        o[n][1] *= alpha;
      }
      m_run = mx;
    }
    const float p0 = m_run == -INFINITY ? 0.f : ex2f(s0 - m_run);
    const float p1 = m_run == -INFINITY ? 0.f : ex2f(s1 - m_run);
    l_part += p0 + p1;
    const uint32_t pa = cvt_bf16x2(p0, p1);
    // O[16 x 256] += P[16 x 8] V[8 x 256]: x4.trans loads bring V rows
    // j0..j0+7, columns 32 h..32 h+31 as four k8 x n8 B fragments
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      uint32_t v0, v1, v2, v3;
      ldsm_x4_t(vt + chunk_off(j0 + (lane & 7), 32 * h + 8 * (lane >> 3)), v0, v1, v2, v3);
      mma1688(o[4 * h], pa, v0);
      mma1688(o[4 * h + 1], pa, v1);
      mma1688(o[4 * h + 2], pa, v2);
      mma1688(o[4 * h + 3], pa, v3);
    }
    __syncthreads();                         // every warp is done with stage s
    ok = sm.timed_out == 0;
    if (ok && t == 0 && i + kStages < n_tiles) issue(i + kStages);
  }
  if (!ok) {
    // Leave without writing (the status word holds PI_ERR_TIMEOUT), after a
    // bounded wait for the copies issued, and after the cluster's barriers.
    if (t == 0)
      for (int i = max(n_tiles - kStages, 0); i < n_tiles; ++i)
        (void)mbar_wait(&sm.full[i % kStages], (i / kStages) & 1, ctl);
    cluster_sync();
    cluster_sync();
    return;
  }

  // ---------------------------------------- warp partials -> CTA partial
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
#pragma unroll
  for (int n = 0; n < 32; ++n)
    *reinterpret_cast<float2*>(&opart[(warp * kDecRows + g) * kDecD + 8 * n + 2 * t4]) =
        make_float2(o[n][0], o[n][1]);
  if (t4 == 0) {
    sm.m[warp][g] = m_run;
    sm.l[warp][g] = l_part;
  }
  __syncthreads();
  // thread t: columns 2t, 2t + 1 of every row; the merged row goes to warp 0's slot
  float Mr[kDecRows], Lr[kDecRows];
  {
    const int d = 2 * t;
    float x[kDecRows][2];
#pragma unroll
    for (int r = 0; r < kDecRows; ++r) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm.m[w][r]);
      float L = 0.f;
      x[r][0] = x[r][1] = 0.f;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float f = M == -INFINITY ? 0.f : ex2f(sm.m[w][r] - M);
        L += f * sm.l[w][r];
        const float2 v = *reinterpret_cast<const float2*>(&opart[(w * kDecRows + r) * kDecD + d]);
        x[r][0] += f * v.x;
        x[r][1] += f * v.y;
      }
      Mr[r] = M;
      Lr[r] = L;
    }
    __syncthreads();                          // all warps' partials are read
#pragma unroll
    for (int r = 0; r < kDecRows; ++r)
      *reinterpret_cast<float2*>(&opart[r * kDecD + d]) = make_float2(x[r][0], x[r][1]);
    if (t == 0) {
#pragma unroll
      for (int r = 0; r < kDecRows; ++r) {
        sm.m[0][r] = Mr[r];
        sm.l[0][r] = Lr[r];
      }
    }
  }
  // --------------------------------- CTA partials -> output, over the cluster
  cluster_sync();
  {
    const int r = t >> 4;                     // 8 rows x 16 threads
    const int d = 32 * (int)crank + 2 * (t & 15);
    const uint32_t o_addr = smem_u32(&opart[r * kDecD + d]);
    const uint32_t m_addr = smem_u32(&sm.m[0][r]);
    const uint32_t l_addr = smem_u32(&sm.l[0][r]);
    float M = -INFINITY;
    float mc[kDecCluster];
#pragma unroll
    for (int c = 0; c < kDecCluster; ++c) {
      mc[c] = ld_cluster_f32(mapa_shared(m_addr, c));
      M = fmaxf(M, mc[c]);
    }
    float L = 0.f, x0 = 0.f, x1 = 0.f;
#pragma unroll
    for (int c = 0; c < kDecCluster; ++c) {
      const float f = M == -INFINITY ? 0.f : ex2f(mc[c] - M);
      L += f * ld_cluster_f32(mapa_shared(l_addr, c));
      x0 += f * ld_cluster_f32(mapa_shared(o_addr, c));
      x1 += f * ld_cluster_f32(mapa_shared(o_addr + 4, c));
    }
    if (r < R) {
      const float inv = L > 0.f ? 1.f / L : 0.f;   // a row that saw nothing writes 0
      *reinterpret_cast<__nv_bfloat162*>(p.out + ((long long)b * R + r) * kDecD + d) =
          __floats2bfloat162_rn(x0 * inv, x1 * inv);
    }
  }
  // no CTA leaves while another may still read its shared memory
  cluster_sync();
}

}  // namespace

bool decode_applies(int Sq, int Hq) { return Sq >= 1 && Sq * Hq <= kDecRows; }

cudaError_t launch_decode(const DecodeParams& p, const DevCtl& ctl, cudaStream_t st) {
  static const cudaError_t attr = cudaFuncSetAttribute(
      decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmemBytes);
  if (attr != cudaSuccess) return attr;
  dim3 grid(kDecCluster, (unsigned)p.B);
  return launch_pdl(decode_kernel, grid, dim3(kDecThreads), kDecSmemBytes, st, p, ctl);
}

}  // namespace piattn

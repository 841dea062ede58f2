// bwd_tc.cu -- gradient of the joint prefill (dq, dk, dv) on tcgen05 tensor
// cores: bf16 inputs, one KV head, head_dim 256.  The training step runs the
// joint forward under gradient ("VLA 代码精读 - OpenPI & StarVLA", 1.5
// Pi0.compute_loss); the pages print no backward, so this is the plain
// derivative of the forward:
//     P = exp(scale * Q K^T - lse)  (the forward's lse; 0 where masked)
//     dP = dO V^T,   D = rowsum(dO * O),   dS = P * (dP - D)
//     dV = P^T dO,   dK = scale * dS^T Q,   dQ = scale * dS K
// over the flattened (token, head) rows of each batch element; with one KV
// head every row reads the same keys.
//
// Tensor memory holds 512 fp32 columns per SM.  At head_dim 256 the dK and dV
// accumulators of one 128-key tile fill it, leaving no room for the score
// tiles a single key-stationary pass would recompute; shared memory likewise
// cannot double-buffer K and V beside a resident Q and dO.  The gradient is
// therefore split into three passes that together run the five contractions
// once each, every one on tcgen05 pair MMAs (cta_group::2, M = 256 rows over a
// cluster of two CTAs):
//
//   score pass  per 256-row tile (query-major): S = Q K^T and dP = dO V^T on
//               64-key tiles into TMEM; one thread per row forms P and dS in
//               fp32 and writes both as bf16 to the caller's workspace
//               [B, rows, Skp] (Skp = S rounded up to 64).
//   dK/dV pass  per 256-key tile (key-major): dV += P^T dO and dK += dS^T Q
//               over 64-row steps, P^T and dS^T read MN-major from the
//               workspace; small problems split the rows into chunks whose
//               partial sums a reduction kernel adds in a fixed order.
//   dQ pass     per 256-row tile: dQ += dS K over the same 64-key tiles.
//
// Tiles are skipped by the forward's rule: a 256-key group is visited by a
// 256-row tile unless no row of it sees any key of the group (block index,
// expert <- FAST, padding).  The score pass writes all four 64-key tiles of a
// visited group (exact zeros where masked), so the dK/dV pass, which reads
// whole groups, never reads an unwritten block.  Everything is deterministic
// (no atomics).  Every wait is bounded (DevCtl) and a timeout is reported in
// the status word.
#include <cfloat>

#include "launch.h"
#include "mask.cuh"

namespace piattn {

namespace {

constexpr int kT = 192;          // warp 0 TMA, warp 1 TMEM + MMA issue, warps 2..5 rows
constexpr int kRows = 128;       // rows per CTA (256 per pair)
constexpr int kD = 256;
constexpr int kKT = 64;          // keys per score tile (32 per CTA)
constexpr int kSup = 256;        // keys per group (4 score tiles; one dK/dV tile)
constexpr int kSmemLimit = 232448;
constexpr int kMaxTiles128 = (kMaxTokens + 127) / 128 + 1;
constexpr float kLog2e = 1.4426950408889634f;

// Shared-memory operand sizes (bf16, 128-byte swizzled [rows x 64] blocks).
constexpr int kRowTile = kRows * kD * 2;       // [128 x 256]   64 KB (Q, dO in the score pass)
constexpr int kItem32 = 32 * kD * 2;           // [32 x 256]    16 KB (this CTA's keys of a score tile)
constexpr int kHalf64 = 64 * 128 * 2;          // [64 x 128]    16 KB (64 rows/keys x this CTA's d-half)
constexpr int kDsTile = kRows * 64 * 2;        // [128 x 64]    16 KB (dS rows of a 64-key tile)

constexpr int kNS1 = 2, kNS2 = 3, kNS3 = 4;    // ring stages per pass
constexpr int kStage1 = 2 * kItem32;           // K, V items
constexpr int kStage2 = 4 * kHalf64;           // P^T, dS^T, dO half, Q half
constexpr int kStage3 = kDsTile + kHalf64;     // dS tile, K half
constexpr int kOps1 = 2 * kRowTile + kNS1 * kStage1;   // 192 KB
constexpr int kOps2 = kNS2 * kStage2;                  // 192 KB
constexpr int kOps3 = kNS3 * kStage3;                  // 128 KB

constexpr uint32_t kIdescScore = idesc_bf16_f32(2 * kRows, kKT, false, false);
constexpr uint32_t kIdescKV = idesc_bf16_f32(2 * kRows, kD, true, true);
constexpr uint32_t kIdescQ = idesc_bf16_f32(2 * kRows, kD, false, true);

struct __align__(8) Ctl {
  uint64_t full[4];       // leader: a ring stage of both CTAs landed
  uint64_t empty[4];      // each CTA: its stage may be refilled
  uint64_t rows_full;     // leader (score pass): Q and dO of both CTAs landed
  uint64_t s_full[2];     // each CTA (score pass): S and dP of a tile in TMEM
  uint64_t s_free[2];     // leader (score pass): the pair's 8 row warps read them
  uint64_t done;          // each CTA: the last accumulation finished
  uint64_t drain;         // leader: every MMA issued has completed
  uint32_t tmem_base;
  int abort;
  int scan[kT / 32];
  uint16_t cs_first[kMaxTiles128];
  uint16_t cs_last[kMaxTiles128];
  uint8_t flags[kMaxTiles128];
};

__host__ __device__ constexpr int ctl_bytes() { return ((int)sizeof(Ctl) + 127) / 128 * 128; }
__host__ __device__ constexpr int pad128(int n) { return (n + 127) / 128 * 128; }
__host__ __device__ constexpr int smem_need(int ops, int S) {
  return ops + ctl_bytes() + pad128(S) * 2;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* abort,
                                              const DevCtl& ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*(volatile int*)abort) return false;
    if ((unsigned long long)(clock64() - t0) > ctl.wait_limit) {
      record_status(ctl, kStatusTimeout);
      *(volatile int*)abort = 1;
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Ctl& c,
                                          const DevCtl& ctl) {
  return __all_sync(0xffffffffu, wait_or_abort(bar, parity, &c.abort, ctl));
}

__device__ __forceinline__ void commit_both(uint64_t* bar) {
  umma_commit_pair(mapa_shared(smem_u32(bar), 0));
  umma_commit_pair(mapa_shared(smem_u32(bar), 1));
}

// Warp-collective: 1 if every token of [tq0, tq1] is an expert (or padding)
// token.
__device__ __forceinline__ bool tokens_all_expert(const uint16_t* codes, int tq0, int tq1,
                                                  int lane) {
  int all_e = 1;
  for (int t = tq0 + lane; t <= tq1; t += 32) all_e &= (codes[t] >> 1) & 1;
  return __all_sync(0xffffffffu, all_e) != 0;
}

// Whether a 256-row tile whose last token has block index csq1 (all of whose
// tokens are expert or padding if all_e) may see a key of the 256-key group
// ks.  False only when no pair of the two can be visible: every key's block
// index is above every row's, the rows are experts and the keys FAST, or the
// keys are all padding.
__device__ __forceinline__ bool group_visible(const Ctl& c, uint32_t csq1, bool all_e, int ks,
                                              int S) {
  const int t0 = 2 * ks;
  const int n128 = (S + 127) / 128;
  if (t0 >= n128) return false;
  if (c.cs_first[t0] > csq1) return false;
  const bool two = t0 + 1 < n128;
  const uint32_t f0 = c.flags[t0], f1 = two ? c.flags[t0 + 1] : 0xFu;
  if ((f0 & 8u) && (f1 & 8u)) return false;                 // all padding
  if (all_e && (f0 & 2u) && (f1 & 2u)) return false;        // experts vs FAST
  return true;
}

// Common prologue: align the shared-memory base, scan the mask into packed
// per-token codes and per-128-token summaries.  Returns nullptr (after
// recording PI_ERR_UNSUPPORTED) if the layout does not fit.
__device__ __forceinline__ uint8_t* bwd_smem(uint8_t* raw, int ops, int S, int smem_bytes,
                                             const DevCtl& ctl) {
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(raw) + 1023) & ~static_cast<uintptr_t>(1023));
  if ((int)(smem - raw) + smem_need(ops, S) > smem_bytes || S > kMaxTokens) {
    if (threadIdx.x == 0) record_status(ctl, kStatusUnsupported);
    return nullptr;
  }
  return smem;
}

// ---------------------------------------------------------------- score pass

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kT, 1)
    bwd_score_kernel(const __grid_constant__ BwdTcParams p, const DevCtl ctl, int smem_bytes) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = bwd_smem(smem_raw, kOps1, p.S, smem_bytes, ctl);
  if (smem == nullptr) return;
  Ctl& c = *reinterpret_cast<Ctl*>(smem + kOps1);
  uint16_t* codes = reinterpret_cast<uint16_t*>(smem + kOps1 + ctl_bytes());
  uint8_t* sQ = smem;
  uint8_t* sdO = smem + kRowTile;
  uint8_t* ring = smem + 2 * kRowTile;

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S, Hq = p.Hq;
  const int rows_per_b = S * Hq;
  const int n_pairs = (rows_per_b + 2 * kRows - 1) / (2 * kRows);
  const int unit = blockIdx.x >> 1;
  const int pair = unit % n_pairs, b = unit / n_pairs;
  const int tok_per_pair = 2 * kRows / Hq;
  const int tq0 = pair * tok_per_pair, tq1 = min(tq0 + tok_per_pair, S) - 1;
  const int row0 = pair * 2 * kRows + (int)rank * kRows;   // this CTA's first row
  const int n_sup = (S + kSup - 1) / kSup;
  const int n_kt = (S + kKT - 1) / kKT;

  const uint8_t* ar_b = p.ar + (long long)b * p.mask_bs;
  const int32_t* seg_b = p.seg ? p.seg + (long long)b * p.mask_bs : nullptr;
  const Flags32 flags0 = load_flags32(ar_b, seg_b, S, (int)threadIdx.x * 32);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS1; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    mbar_init(&c.rows_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&c.s_full[s], 1);
      mbar_init(&c.s_free[s], 8);
    }
    mbar_init(&c.drain, 1);
    c.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&p.map_q);
    tma_prefetch_desc(&p.map_do);
    tma_prefetch_desc(&p.map_k32);
    tma_prefetch_desc(&p.map_v32);
  }
  cluster_sync();
  // Q and dO of this CTA's 128 rows load during the mask scan.
  const uint32_t rows_full_l = mapa_shared(smem_u32(&c.rows_full), 0);
  if (threadIdx.x == 0) {
    if (leader) mbar_arrive_expect_tx(&c.rows_full, 4 * kRowTile);
    tma_load_4d_pair(sQ, &p.map_q, rows_full_l, 0, row0, 0, b);
    tma_load_4d_pair(sdO, &p.map_do, rows_full_l, 0, row0, 0, b);
  }
  if (warp == 1) {
    tmem_alloc_pair(&c.tmem_base, 256);
    tmem_relinquish_pair();
  }
  build_codes_x32<kT>(ar_b, seg_b, S, pad128(S), codes, c.scan, flags0,
                      TileSums{c.cs_first, c.cs_last, c.flags});
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  const uint32_t csq1 = codes[tq1] >> 2;
  const bool all_e = tokens_all_expert(codes, tq0, tq1, lane);

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    uint32_t n = 0;
    bool ok = true;
    for (int ks = 0; ks < n_sup && ok; ++ks) {
      if (!group_visible(c, csq1, all_e, ks, S)) continue;
      for (int kt = 4 * ks; kt < min(4 * ks + 4, n_kt) && ok; ++kt, ++n) {
        const int s = (int)(n % kNS1);
        const uint32_t rel = n / kNS1;
        if (rel > 0 && !warp_wait(&c.empty[s], (rel - 1) & 1, c, ctl)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t full_l = mapa_shared(smem_u32(&c.full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&c.full[s], 2 * kStage1);
          uint8_t* st = ring + s * kStage1;
          // this CTA's 32 keys of the tile, all 256 columns, of K and of V
          tma_load_4d_pair(st, &p.map_k32, full_l, 0, kt * kKT + 32 * (int)rank, 0, b);
          tma_load_4d_pair(st + kItem32, &p.map_v32, full_l, 0, kt * kKT + 32 * (int)rank, 0, b);
        }
        __syncwarp();
      }
    }
    // Loads complete on the leader's barriers: wait there (bounded) for the
    // last phase of each, so no copy is in flight when the cluster leaves.
    if (leader && lane == 0) {
      (void)mbar_wait(&c.rows_full, 0, ctl);
      for (int s = 0; s < kNS1; ++s) {
        const uint32_t n_s = n > (uint32_t)s ? (n - (uint32_t)s + kNS1 - 1) / kNS1 : 0;
        if (n_s > 0) (void)mbar_wait(&c.full[s], (n_s - 1) & 1, ctl);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------- MMA issue (leader CTA only)
    if (leader) {
      const uint64_t qdesc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dodesc = sdesc_sw128(smem_u32(sdO), 16, 1024);
      const uint64_t rdesc = sdesc_sw128(smem_u32(ring), 16, 1024);
      uint32_t n = 0;
      bool ok = warp_wait(&c.rows_full, 0, c, ctl);
      for (int ks = 0; ks < n_sup && ok; ++ks) {
        if (!group_visible(c, csq1, all_e, ks, S)) continue;
        for (int kt = 4 * ks; kt < min(4 * ks + 4, n_kt) && ok; ++kt, ++n) {
          const int s = (int)(n % kNS1);
          if (!warp_wait(&c.full[s], (n / kNS1) & 1, c, ctl)) { ok = false; break; }
          // S/dP buffer n % 2 was last read by the row warps at tile n - 2.
          if (n >= 2 && !warp_wait(&c.s_free[n & 1], ((n - 2) >> 1) & 1, c, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint64_t kd = rdesc + (uint64_t)((s * kStage1) >> 4);
            const uint64_t vd = rdesc + (uint64_t)((s * kStage1 + kItem32) >> 4);
            const uint32_t tS = tmem + 64 * (n & 1), tP = tmem + 128 + 64 * (n & 1);
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              // A: [128 rows x 16 d] of Q / dO; B: [32 keys x 16 d] of K / V; both
              // K-major, 8-row groups 1024 B apart, a K step walks 32 B inside a
              // 64-column block, then to the next block.
              const uint32_t aoff = (uint32_t)((kk >> 2) * (kRows * 128) + (kk & 3) * 32);
              const uint32_t boff = (uint32_t)((kk >> 2) * (32 * 128) + (kk & 3) * 32);
              umma_pair_ss(tS, qdesc + (aoff >> 4), kd + (boff >> 4), kIdescScore,
                           kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint32_t aoff = (uint32_t)((kk >> 2) * (kRows * 128) + (kk & 3) * 32);
              const uint32_t boff = (uint32_t)((kk >> 2) * (32 * 128) + (kk & 3) * 32);
              umma_pair_ss(tP, dodesc + (aoff >> 4), vd + (boff >> 4), kIdescScore,
                           kk > 0 ? 1u : 0u);
            }
            commit_both(&c.empty[s]);
            commit_both(&c.s_full[n & 1]);
          }
          __syncwarp();
        }
      }
      if (lane == 0) umma_commit_pair(smem_u32(&c.drain));
      __syncwarp();
      (void)mbar_wait(&c.drain, 0, ctl);
    }
  } else {
    // ------------------------------------------ row warps (both CTAs)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int rho = row0 + r;
    const bool row_valid = rho < rows_per_b;
    const int tok = row_valid ? rho / Hq : tq1;
    const uint32_t cq = codes[tok];
    const uint32_t csq = cq >> 2;
    const bool row_expert = (cq & 2u) != 0;
    const bool row_live = row_valid && !is_pad(cq);
    const long long grow = (long long)b * rows_per_b + (row_valid ? rho : 0);
    const float lse2 = row_live ? p.lse[grow] * kLog2e : 0.f;
    const float Dv = row_live ? p.D[grow] : 0.f;
    const float cs = p.scale_log2;
    __nv_bfloat16* prow = p.P + grow * p.Skp;
    __nv_bfloat16* dsrow = p.dS + grow * p.Skp;
    const uint32_t s_free_l0 = mapa_shared(smem_u32(&c.s_free[0]), 0);
    const uint32_t s_free_l1 = mapa_shared(smem_u32(&c.s_free[1]), 0);
    uint32_t n = 0;
    bool ok = true;
    for (int ks = 0; ks < n_sup && ok; ++ks) {
      if (!group_visible(c, csq1, all_e, ks, S)) continue;
      for (int kt = 4 * ks; kt < min(4 * ks + 4, n_kt) && ok; ++kt, ++n) {
        const int bs = (int)(n & 1);
        const int k0 = kt * kKT;
        // Keys of this tile the row sees: a prefix (block index is
        // non-decreasing), minus FAST keys for expert rows and padding keys.
        int e = 0;
#pragma unroll
        for (int step = kKT; step >= 1; step >>= 1) {
          const int probe = e + step;
          if (probe <= kKT && (uint32_t)(codes[k0 + probe - 1] >> 2) <= csq) e = probe;
        }
        e = row_live ? min(e, S - k0) : 0;
        const uint32_t tf = c.flags[kt >> 1];
        const bool hole = ((tf & 1u) && row_expert) || (tf & 4u);
        if (!warp_wait(&c.s_full[bs], (n >> 1) & 1, c, ctl)) { ok = false; break; }
        tc_fence_after();
        uint32_t s0[32], s1[32], d0[32], d1[32];
        tmem_ld32(tmem + lane_off + 64 * bs, s0);
        tmem_ld32(tmem + lane_off + 64 * bs + 32, s1);
        tmem_ld32(tmem + lane_off + 128 + 64 * bs, d0);
        tmem_ld32(tmem + lane_off + 128 + 64 * bs + 32, d1);
        tmem_ld_wait();
        reg_fence(s0);
        reg_fence(s1);
        reg_fence(d0);
        reg_fence(d1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(bs ? s_free_l1 : s_free_l0);
        uint32_t hid0 = 0u, hid1 = 0u;   // bit j: key j of the tile hidden by the hole rule
        if (hole) {
          const uint4* kc = reinterpret_cast<const uint4*>(codes + k0);
#pragma unroll
          for (int q8 = 0; q8 < kKT / 8; ++q8) {
            const uint4 v4 = kc[q8];
            const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
            for (int h = 0; h < 8; ++h) {
              const int j = 8 * q8 + h;
              const uint32_t ck = (wv[h >> 1] >> (16 * (h & 1))) & 0xFFFFu;
              const uint32_t hide = ((row_expert && (ck & 1u)) || is_pad(ck)) ? 1u : 0u;
              if (j < 32) hid0 |= hide << j;
              else hid1 |= hide << (j - 32);
            }
          }
        }
        uint32_t pk[32], dk[32];
#pragma unroll
        for (int j = 0; j < kKT; j += 2) {
          float sv0 = __uint_as_float(j < 32 ? s0[j] : s1[j - 32]);
          float sv1 = __uint_as_float(j + 1 < 32 ? s0[j + 1] : s1[j - 31]);
          const float dv0 = __uint_as_float(j < 32 ? d0[j] : d1[j - 32]);
          const float dv1 = __uint_as_float(j + 1 < 32 ? d0[j + 1] : d1[j - 31]);
          const uint32_t h0 = j < 32 ? (hid0 >> j) & 1u : (hid1 >> (j - 32)) & 1u;
          const uint32_t h1 = j + 1 < 32 ? (hid0 >> (j + 1)) & 1u : (hid1 >> (j - 31)) & 1u;
          const float2 t = ffma2(make_float2(sv0, sv1), make_float2(cs, cs),
                                 make_float2(-lse2, -lse2));
          const float p0 = (j < e && !h0) ? ex2(t.x) : 0.f;
          const float p1 = (j + 1 < e && !h1) ? ex2(t.y) : 0.f;
          pk[j >> 1] = cvt_bf16x2(p0, p1);
          dk[j >> 1] = cvt_bf16x2(p0 * (dv0 - Dv), p1 * (dv1 - Dv));
        }
        if (row_valid) {
          uint4* pd = reinterpret_cast<uint4*>(prow + k0);
          uint4* dd = reinterpret_cast<uint4*>(dsrow + k0);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            pd[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            dd[q] = make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 256);
  }
}

// ----------------------------------------------------- epilogue helpers

// Warp-collective: this thread's TMEM row (256 fp32 columns from `col`) times
// `mul` to dst[0..255] (fp32, 16-byte aligned) when `store`; zeros when `zero`
// (no TMEM read then).
__device__ __forceinline__ void tmem_row_out(uint32_t taddr, float mul, float* dst, bool store,
                                             bool zero) {
#pragma unroll 1
  for (int cc = 0; cc < kD / 32; ++cc) {
    uint32_t o[32];
    if (!zero) {
      tmem_ld32(taddr + 32 * cc, o);
      tmem_ld_wait();
      reg_fence(o);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = 0u;
    }
    if (store) {
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(dst + 32 * cc + e) =
            make_float4(__uint_as_float(o[e]) * mul, __uint_as_float(o[e + 1]) * mul,
                        __uint_as_float(o[e + 2]) * mul, __uint_as_float(o[e + 3]) * mul);
    }
  }
}

// ------------------------------------------------------------- dK/dV pass

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kT, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ BwdTcParams p, const DevCtl ctl, int smem_bytes) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = bwd_smem(smem_raw, kOps2, p.S, smem_bytes, ctl);
  if (smem == nullptr) return;
  Ctl& c = *reinterpret_cast<Ctl*>(smem + kOps2);
  uint16_t* codes = reinterpret_cast<uint16_t*>(smem + kOps2 + ctl_bytes());
  uint8_t* ring = smem;

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S, Hq = p.Hq;
  const int rows_per_b = S * Hq;
  const int n_pairs = (rows_per_b + 2 * kRows - 1) / (2 * kRows);
  const int n_sup = (S + kSup - 1) / kSup;
  const int unit = blockIdx.x >> 1;
  const int chunk = unit % p.n_chunks;
  const int ks = (unit / p.n_chunks) % n_sup;
  const int b = unit / p.n_chunks / n_sup;
  const int p_begin = chunk * p.pairs_per_chunk;
  const int p_end = min(p_begin + p.pairs_per_chunk, n_pairs);
  const int tok_per_pair = 2 * kRows / Hq;

  const uint8_t* ar_b = p.ar + (long long)b * p.mask_bs;
  const int32_t* seg_b = p.seg ? p.seg + (long long)b * p.mask_bs : nullptr;
  const Flags32 flags0 = load_flags32(ar_b, seg_b, S, (int)threadIdx.x * 32);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS2; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    mbar_init(&c.done, 1);
    mbar_init(&c.drain, 1);
    c.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&p.map_pT);
    tma_prefetch_desc(&p.map_dsT);
    tma_prefetch_desc(&p.map_qh);
    tma_prefetch_desc(&p.map_doh);
  }
  cluster_sync();
  if (warp == 1) {
    tmem_alloc_pair(&c.tmem_base, 512);
    tmem_relinquish_pair();
  }
  build_codes_x32<kT>(ar_b, seg_b, S, pad128(S), codes, c.scan, flags0,
                      TileSums{c.cs_first, c.cs_last, c.flags});
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  const uint32_t tdV = tmem, tdK = tmem + 256;

  // The 64-row steps of this unit: every step of each row tile in
  // [p_begin, p_end) that may see a key of group ks (the same rule the score
  // pass used to decide which groups it wrote).
  auto tile_steps = [&](int pt) -> int {
    const int tq0 = pt * tok_per_pair, tq1 = min(tq0 + tok_per_pair, S) - 1;
    const bool all_e = tokens_all_expert(codes, tq0, tq1, lane);
    if (!group_visible(c, (uint32_t)(codes[tq1] >> 2), all_e, ks, S)) return 0;
    return (min(2 * kRows, rows_per_b - pt * 2 * kRows) + 63) / 64;
  };

  uint32_t n_total = 0;     // steps this unit runs (each role counts them)
  if (warp == 0) {
    // ---------------------------------------------------------- producer
    bool ok = true;
    for (int pt = p_begin; pt < p_end && ok; ++pt) {
      const int nst = tile_steps(pt);
      for (int st = 0; st < nst && ok; ++st, ++n_total) {
        const uint32_t n = n_total;
        const int s = (int)(n % kNS2);
        const uint32_t rel = n / kNS2;
        if (rel > 0 && !warp_wait(&c.empty[s], (rel - 1) & 1, c, ctl)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t full_l = mapa_shared(smem_u32(&c.full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&c.full[s], 2 * kStage2);
          uint8_t* sg = ring + s * kStage2;
          const int r0 = pt * 2 * kRows + 64 * st;
          const int kb = 4 * ks + 2 * (int)rank;       // this CTA's 128 keys: 2 blocks of 64
          tma_load_4d_pair(sg, &p.map_pT, full_l, 0, r0, kb, b);
          tma_load_4d_pair(sg + kHalf64, &p.map_dsT, full_l, 0, r0, kb, b);
          tma_load_4d_pair(sg + 2 * kHalf64, &p.map_doh, full_l, 0, r0, 2 * (int)rank, b);
          tma_load_4d_pair(sg + 3 * kHalf64, &p.map_qh, full_l, 0, r0, 2 * (int)rank, b);
        }
        __syncwarp();
      }
    }
    if (leader && lane == 0) {
      for (int s = 0; s < kNS2; ++s) {
        const uint32_t n_s = n_total > (uint32_t)s ? (n_total - (uint32_t)s + kNS2 - 1) / kNS2 : 0;
        if (n_s > 0) (void)mbar_wait(&c.full[s], (n_s - 1) & 1, ctl);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------- MMA issue (leader CTA only)
    for (int pt = p_begin; pt < p_end; ++pt) n_total += (uint32_t)tile_steps(pt);
    if (leader) {
      const uint64_t rdesc = sdesc_sw128(smem_u32(ring), kHalf64 / 2, 1024);
      uint32_t n = 0;
      bool ok = true;
      for (; n < n_total && ok; ++n) {
        const int s = (int)(n % kNS2);
        if (!warp_wait(&c.full[s], (n / kNS2) & 1, c, ctl)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t base = (uint32_t)(s * kStage2);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            // A = P^T / dS^T [128 keys x 16 rows] per CTA, B = dO / Q [16 rows x
            // (128 columns per CTA)], both MN-major: 8-row groups 1024 B apart,
            // 64-wide blocks 8 KB apart; a K step is 16 rows (2048 B).
            const uint32_t ko = (uint32_t)(k4 * 2048);
            umma_pair_ss(tdV, rdesc + ((base + ko) >> 4),
                         rdesc + ((base + 2 * kHalf64 + ko) >> 4), kIdescKV,
                         (n > 0 || k4 > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint32_t ko = (uint32_t)(k4 * 2048);
            umma_pair_ss(tdK, rdesc + ((base + kHalf64 + ko) >> 4),
                         rdesc + ((base + 3 * kHalf64 + ko) >> 4), kIdescKV,
                         (n > 0 || k4 > 0) ? 1u : 0u);
          }
          commit_both(&c.empty[s]);
          if (n + 1 == n_total) commit_both(&c.done);
        }
        __syncwarp();
      }
      if (lane == 0) umma_commit_pair(smem_u32(&c.drain));
      __syncwarp();
      (void)mbar_wait(&c.drain, 0, ctl);
    }
  } else {
    // ------------------------------------ epilogue warps (both CTAs)
    for (int pt = p_begin; pt < p_end; ++pt) n_total += (uint32_t)tile_steps(pt);
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int key = ks * kSup + (int)rank * kRows + r;
    const bool have = n_total > 0;
    bool ok = true;
    if (have) {
      ok = warp_wait(&c.done, 0, c, ctl);
      tc_fence_after();
    }
    if (ok) {
      float* dkdst;
      float* dvdst;
      bool store;
      if (p.n_chunks == 1) {
        store = key < S;
        const long long o = ((long long)b * S + (store ? key : 0)) * kD;
        dkdst = p.dk + o;
        dvdst = p.dv + o;
      } else {
        store = true;
        const long long kpad = (long long)n_sup * kSup;
        const long long o = (((long long)chunk * p.B + b) * kpad + key) * kD;
        dkdst = p.part + o;
        dvdst = p.part + (long long)p.n_chunks * p.B * kpad * kD + o;
      }
      tmem_row_out(tdK + lane_off, p.scale, dkdst, store, !have);
      tmem_row_out(tdV + lane_off, 1.f, dvdst, store, !have);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ----------------------------------------------------------------- dQ pass

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kT, 1)
    bwd_dq_tc_kernel(const __grid_constant__ BwdTcParams p, const DevCtl ctl, int smem_bytes) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = bwd_smem(smem_raw, kOps3, p.S, smem_bytes, ctl);
  if (smem == nullptr) return;
  Ctl& c = *reinterpret_cast<Ctl*>(smem + kOps3);
  uint16_t* codes = reinterpret_cast<uint16_t*>(smem + kOps3 + ctl_bytes());
  uint8_t* ring = smem;

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S, Hq = p.Hq;
  const int rows_per_b = S * Hq;
  const int n_pairs = (rows_per_b + 2 * kRows - 1) / (2 * kRows);
  const int unit = blockIdx.x >> 1;
  const int pair = unit % n_pairs, b = unit / n_pairs;
  const int tok_per_pair = 2 * kRows / Hq;
  const int tq0 = pair * tok_per_pair, tq1 = min(tq0 + tok_per_pair, S) - 1;
  const int row0 = pair * 2 * kRows + (int)rank * kRows;
  const int n_sup = (S + kSup - 1) / kSup;
  const int n_kt = (S + kKT - 1) / kKT;

  const uint8_t* ar_b = p.ar + (long long)b * p.mask_bs;
  const int32_t* seg_b = p.seg ? p.seg + (long long)b * p.mask_bs : nullptr;
  const Flags32 flags0 = load_flags32(ar_b, seg_b, S, (int)threadIdx.x * 32);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS3; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    mbar_init(&c.done, 1);
    mbar_init(&c.drain, 1);
    c.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&p.map_ds);
    tma_prefetch_desc(&p.map_kh);
  }
  cluster_sync();
  if (warp == 1) {
    tmem_alloc_pair(&c.tmem_base, 256);
    tmem_relinquish_pair();
  }
  build_codes_x32<kT>(ar_b, seg_b, S, pad128(S), codes, c.scan, flags0,
                      TileSums{c.cs_first, c.cs_last, c.flags});
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  const uint32_t csq1 = codes[tq1] >> 2;
  const bool all_e = tokens_all_expert(codes, tq0, tq1, lane);
  uint32_t n_total = 0;
  for (int ks = 0; ks < n_sup; ++ks)
    if (group_visible(c, csq1, all_e, ks, S)) n_total += (uint32_t)(min(4 * ks + 4, n_kt) - 4 * ks);

  if (warp == 0) {
    uint32_t n = 0;
    bool ok = true;
    for (int ks = 0; ks < n_sup && ok; ++ks) {
      if (!group_visible(c, csq1, all_e, ks, S)) continue;
      for (int kt = 4 * ks; kt < min(4 * ks + 4, n_kt) && ok; ++kt, ++n) {
        const int s = (int)(n % kNS3);
        const uint32_t rel = n / kNS3;
        if (rel > 0 && !warp_wait(&c.empty[s], (rel - 1) & 1, c, ctl)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t full_l = mapa_shared(smem_u32(&c.full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&c.full[s], 2 * kStage3);
          uint8_t* sg = ring + s * kStage3;
          tma_load_4d_pair(sg, &p.map_ds, full_l, 0, row0, kt, b);
          tma_load_4d_pair(sg + kDsTile, &p.map_kh, full_l, 0, kt * kKT, 2 * (int)rank, b);
        }
        __syncwarp();
      }
    }
    if (leader && lane == 0) {
      for (int s = 0; s < kNS3; ++s) {
        const uint32_t n_s = n > (uint32_t)s ? (n - (uint32_t)s + kNS3 - 1) / kNS3 : 0;
        if (n_s > 0) (void)mbar_wait(&c.full[s], (n_s - 1) & 1, ctl);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (leader) {
      const uint64_t adesc = sdesc_sw128(smem_u32(ring), 16, 1024);
      const uint64_t bdesc = sdesc_sw128(smem_u32(ring), kHalf64 / 2, 1024);
      uint32_t n = 0;
      bool ok = true;
      for (; n < n_total && ok; ++n) {
        const int s = (int)(n % kNS3);
        if (!warp_wait(&c.full[s], (n / kNS3) & 1, c, ctl)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t base = (uint32_t)(s * kStage3);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            // A = dS [128 rows x 16 keys] K-major (a K step walks 32 B of the
            // 128-byte line); B = K [16 keys x (128 columns per CTA)] MN-major.
            umma_pair_ss(tmem, adesc + ((base + k4 * 32) >> 4),
                         bdesc + ((base + kDsTile + k4 * 2048) >> 4), kIdescQ,
                         (n > 0 || k4 > 0) ? 1u : 0u);
          }
          commit_both(&c.empty[s]);
          if (n + 1 == n_total) commit_both(&c.done);
        }
        __syncwarp();
      }
      if (lane == 0) umma_commit_pair(smem_u32(&c.drain));
      __syncwarp();
      (void)mbar_wait(&c.drain, 0, ctl);
    }
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int rho = row0 + r;
    const bool row_valid = rho < rows_per_b;
    const bool have = n_total > 0;
    bool ok = true;
    if (have) {
      ok = warp_wait(&c.done, 0, c, ctl);
      tc_fence_after();
    }
    if (ok) {
      float* dst = p.dq + ((long long)b * rows_per_b + (row_valid ? rho : 0)) * kD;
      tmem_row_out(tmem + lane_off, p.scale, dst, row_valid, !have);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 256);
  }
}

// ------------------------------------------------------- small kernels

// D[row] = sum_d dO[row, d] * O[row, d] in fp32: one warp per row, each lane
// 8 of the 256 columns (16-byte loads).
__global__ void __launch_bounds__(256)
    bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ out,
                      const __nv_bfloat16* __restrict__ dout, float* __restrict__ D,
                      long long n_rows) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < n_rows; row += warps) {
    const uint4 a = reinterpret_cast<const uint4*>(out + row * kD)[lane];
    const uint4 g = reinterpret_cast<const uint4*>(dout + row * kD)[lane];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[i]));
      const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[i]));
      s = fmaf(af.x, gf.x, s);
      s = fmaf(af.y, gf.y, s);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) D[row] = s;
  }
}

// dk, dv = the sums over row chunks of the dK/dV pass's partials, added in
// chunk order (deterministic).
__global__ void __launch_bounds__(256)
    bwd_chunk_sum_kernel(const float* __restrict__ part, float* __restrict__ dk,
                         float* __restrict__ dv, int n_chunks, int B, int S, int kpad) {
  const long long n4 = (long long)B * S * (kD / 4);
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long per_chunk = (long long)B * kpad * kD;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const long long c4 = i % (kD / 4);
    const long long bk = i / (kD / 4);            // b * S + key
    const long long b = bk / S, key = bk - b * S;
    const long long o = (b * kpad + key) * kD + 4 * c4;
    float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = sk;
    for (int ch = 0; ch < n_chunks; ++ch) {
      const float4 a = *reinterpret_cast<const float4*>(part + ch * per_chunk + o);
      const float4 v = *reinterpret_cast<const float4*>(part + (n_chunks + ch) * per_chunk + o);
      sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
      sv.x += v.x; sv.y += v.y; sv.z += v.z; sv.w += v.w;
    }
    reinterpret_cast<float4*>(dk)[i] = sk;
    reinterpret_cast<float4*>(dv)[i] = sv;
  }
}

template <typename K>
cudaError_t launch_cluster_kernel(K kernel, int clusters, int ops, const BwdTcParams& p,
                                  const DevCtl& ctl, cudaStream_t st) {
  static_assert(sizeof(BwdTcParams) <= 4096, "kernel parameters too large");
  const int smem = min(smem_need(ops, p.S) + 1024, kSmemLimit);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemLimit);
  if (e != cudaSuccess) return e;
  kernel<<<2 * clusters, kT, smem, st>>>(p, ctl, smem);
  return cudaGetLastError();
}

}  // namespace

BwdTcPlan bwd_tc_plan(int B, int S, int Hq, int sms) {
  BwdTcPlan pl{};
  const int rows = S * Hq;
  pl.n_pairs = (rows + 2 * kRows - 1) / (2 * kRows);
  pl.n_sup = (S + kSup - 1) / kSup;
  pl.Skp = (S + kKT - 1) / kKT * kKT;
  // Row chunks of the dK/dV pass: the fewest that keep the SM pairs as busy
  // as any larger count would (whole waves of clusters).
  const int clusters = max(sms / 2, 1);
  const long long units = (long long)B * pl.n_sup;
  int best = 1;
  double best_t = 1e30;
  for (int c = 1; c <= pl.n_pairs && c <= 64; ++c) {
    const int ppc = (pl.n_pairs + c - 1) / c;
    const int cc = (pl.n_pairs + ppc - 1) / ppc;                  // chunks actually used
    const double waves = (double)((units * cc + clusters - 1) / clusters);
    const double t = waves * ppc;
    if (t < best_t - 1e-9) {
      best_t = t;
      best = cc;
    }
  }
  pl.pairs_per_chunk = (pl.n_pairs + best - 1) / best;
  pl.n_chunks = (pl.n_pairs + pl.pairs_per_chunk - 1) / pl.pairs_per_chunk;
  const size_t a = 256;
  auto up = [&](size_t x) { return (x + a - 1) / a * a; };
  pl.off_D = 0;
  pl.off_P = up((size_t)B * rows * sizeof(float));
  pl.off_dS = pl.off_P + up((size_t)B * rows * pl.Skp * 2);
  pl.off_part = pl.off_dS + up((size_t)B * rows * pl.Skp * 2);
  const size_t part = pl.n_chunks > 1
                          ? (size_t)2 * pl.n_chunks * B * pl.n_sup * kSup * kD * sizeof(float)
                          : 0;
  pl.bytes = pl.off_part + up(part);
  return pl;
}

cudaError_t launch_backward_tc(const BwdTcParams& p, const DevCtl& ctl, cudaStream_t st) {
  const long long rows = (long long)p.B * p.S * p.Hq;
  const int rd_blocks = (int)min((rows + 7) / 8, (long long)148 * 16);
  bwd_rowdot_kernel<<<rd_blocks, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(p.out), static_cast<const __nv_bfloat16*>(p.dout),
      const_cast<float*>(p.D), rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n_pairs = (p.S * p.Hq + 2 * kRows - 1) / (2 * kRows);
  const int n_sup = (p.S + kSup - 1) / kSup;
  e = launch_cluster_kernel(bwd_score_kernel, p.B * n_pairs, kOps1, p, ctl, st);
  if (e != cudaSuccess) return e;
  e = launch_cluster_kernel(bwd_dkdv_tc_kernel, p.B * n_sup * p.n_chunks, kOps2, p, ctl, st);
  if (e != cudaSuccess) return e;
  if (p.n_chunks > 1) {
    const long long n4 = (long long)p.B * p.S * (kD / 4);
    const int blocks = (int)min((n4 + 255) / 256, (long long)148 * 8);
    bwd_chunk_sum_kernel<<<blocks, 256, 0, st>>>(p.part, p.dk, p.dv, p.n_chunks, p.B, p.S,
                                                 n_sup * kSup);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return launch_cluster_kernel(bwd_dq_tc_kernel, p.B * n_pairs, kOps3, p, ctl, st);
}

}  // namespace piattn

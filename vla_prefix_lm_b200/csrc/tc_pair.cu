// tc_pair.cu -- bf16 joint (prefix-LM) attention on tcgen05, CTA-pair (2-SM) form.
//
// A cluster of two CTAs computes one 256-row query tile: 256 / Hq query
// tokens x Hq heads, 128 rows per CTA.  With a single KV head all rows read
// the same K/V rows ("π0.5 vs MM-DiT joint attention", "joint attention 只管
// 算子": 8 query heads, 1 KV head, head_dim 256, one shared KV pool).
//
// Per key tile of 128 keys, issued by ONE thread of the even CTA for the pair:
//   S = Q K^T   tcgen05.mma.cta_group::2, M = 256: A = Q rows of each CTA
//               (its shared memory), B = K split by keys (64 per CTA)
//   P           fp32 online softmax in each CTA, one thread per row
//   O += P V    tcgen05.mma.cta_group::2: A = P (each CTA's TMEM, bf16),
//               B = V split by columns (128 of the 256 per CTA)
// Each SM therefore streams half of every K/V tile (32 B/clk at the full
// tensor rate instead of 64), and every MMA instruction and every barrier
// round trip covers twice the work of a one-CTA, 64-key design.
//
// Mask: every CTA scans ar_mask / segment_ids into packed per-token codes
// (mask.cuh), classifies each key tile for the whole 256-row pair tile (skip /
// full / partial; both CTAs reach the same list), and masks a partial tile per
// row by its visible-prefix length plus, for expert rows, the FAST keys.  No
// mask is materialised.
//
// Warp roles per CTA (192 threads):
//   warp 0      TMA producer for this CTA's halves (both CTAs)
//   warp 1      TMEM allocation (both CTAs, cta_group::2); MMA issue (even CTA)
//   warps 2..5  softmax, O correction, epilogue (both CTAs, own rows)
//
// TMEM per CTA (512 columns): O fp32 [0,256) | S0 [256,384) | S1 [384,512);
// P of tile t is packed bf16 over the first 64 columns of S[t%2].
// Shared memory per CTA: Q 64 KB | ring 4 x 32 KB (K halves [64 x 256], V
// halves [128 x 128]) | control | per-token codes.  The epilogue stages the
// bf16 output in the Q area (dead after the last QK).
//
// Synchronisation across the pair: the even CTA owns q_full, kv_full and
// p_full (the odd CTA's TMA loads and softmax warps arrive there through
// cluster addresses); the MMA thread's commits arrive on the s_full, o_done
// and kv_empty barriers of both CTAs.  Every wait is bounded (DevCtl).
#include <cfloat>

#include "launch.h"
#include "mask.cuh"

namespace piattn {

namespace {

constexpr int kThreads = 192;
constexpr int kBM = 128;                    // query rows per CTA (256 per pair)
constexpr int kBN = 128;                    // keys per key tile
constexpr int kD = 256;
constexpr int kQBlk = kBM * 128;            // [128 rows x 64 bf16] = 16 KB
constexpr int kQBytes = 4 * kQBlk;          // 64 KB
constexpr int kKBlk = 64 * 128;             // K half block: [64 keys x 64 d] = 8 KB
constexpr int kVBlk = kBN * 128;            // V half block: [128 keys x 64 d] = 16 KB
constexpr int kItemBytes = 32768;           // K half (4 x 8 KB) or V half (2 x 16 KB)
constexpr int kStages = 4;
constexpr int kOffQ = 0;
constexpr int kOffRing = kQBytes;
constexpr int kOffCtl = kOffRing + kStages * kItemBytes;
constexpr int kMaxKeyTiles = (kMaxTokens + kBN - 1) / kBN + 2;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: P stays <= 256

constexpr uint32_t kIdescQK = idesc_bf16_f32(2 * kBM, kBN, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(2 * kBM, kD, false, true);
constexpr uint32_t kColO = 0, kColS = 256;

constexpr uint16_t kTilePartial = 0x8000;
constexpr uint16_t kTileAnyFast = 0x4000;
constexpr uint16_t kTileIndex = 0x3FFF;

struct __align__(8) Smem {
  uint64_t q_full;               // even CTA: both Q halves landed
  uint64_t kv_full[kStages];     // even CTA: both halves of a K or V item landed
  uint64_t kv_empty[kStages];    // each CTA: its ring stage may be refilled
  uint64_t s_full[2];            // each CTA: S tile in its TMEM
  uint64_t p_full[2];            // even CTA: P written by the pair's 8 softmax warps
  uint64_t o_done;               // each CTA: PV finished
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_list;
  int scan[kThreads / 32];
  uint16_t list[kMaxKeyTiles];
  uint16_t tile_cs_first[kMaxKeyTiles];
  uint16_t tile_cs_last[kMaxKeyTiles];
  uint8_t tile_fast[kMaxKeyTiles];
};

constexpr int kOffCodes = kOffCtl + ((int)sizeof(Smem) + 127) / 128 * 128;

__host__ __device__ constexpr int pad_tokens(int n) { return (n + 127) / 128 * 128; }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Smem& sm,
                                              const DevCtl& ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*(volatile int*)&sm.abort) return false;
    if ((unsigned long long)(clock64() - t0) > ctl.wait_limit) {
      record_status(ctl, kStatusTimeout);
      *(volatile int*)&sm.abort = 1;
      return false;
    }
  }
  return true;
}

struct KvTile {
  int src;       // 0: k/v (prefill keys or suffix keys), 1: cached prefix
  int tile;
  bool partial;
  bool any_fast;
};

template <bool kSuffix>
__device__ __forceinline__ KvTile kv_tile_at(const Smem& sm, int idx, int n_cache, int P) {
  if (kSuffix && idx < n_cache) return KvTile{1, idx, (idx + 1) * kBN > P, false};
  const uint16_t e = sm.list[kSuffix ? idx - n_cache : idx];
  return KvTile{0, (int)(e & kTileIndex), (e & kTilePartial) != 0, (e & kTileAnyFast) != 0};
}

template <bool kSuffix>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tc_pair_kernel(const __grid_constant__ TcParams p, const DevCtl ctl) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Smem& sm = *reinterpret_cast<Smem*>(smem + kOffCtl);
  uint16_t* codes = reinterpret_cast<uint16_t*>(smem + kOffCodes);
  uint8_t* sQ = smem + kOffQ;
  uint8_t* ring = smem + kOffRing;

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_per_b = p.Sq * p.Hq;
  const int n_pairs = (rows_per_b + 2 * kBM - 1) / (2 * kBM);
  const int pair = (blockIdx.x >> 1) % n_pairs;
  const int split = (blockIdx.x >> 1) / n_pairs;
  const int b = blockIdx.y;
  const int row0 = pair * 2 * kBM + (int)rank * kBM;   // first row of this CTA
  const int tok_per_pair = 2 * kBM / p.Hq;
  const int tq0 = pair * tok_per_pair;                  // first token of the pair
  const int tq1 = min(tq0 + tok_per_pair, p.Sq) - 1;    // last valid token of the pair
  const int n_key_tok = p.Sq;
  const int n_cache = kSuffix ? (p.P + kBN - 1) / kBN : 0;

  // The mask bytes are the first global reads: issue them before anything
  // else so their latency hides behind the barrier and TMEM set-up.
  const uint8_t* ar_b = p.ar + (long long)b * p.mask_bs;
  const int32_t* seg_b = (!kSuffix && p.seg) ? p.seg + (long long)b * p.mask_bs : nullptr;
  const Flags32 flags0 = load_flags32(ar_b, seg_b, n_key_tok, (int)threadIdx.x * 32);

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 8);
    }
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&p.map_q);
    tma_prefetch_desc(&p.map_k);
    tma_prefetch_desc(&p.map_vh);
    if (kSuffix) {
      tma_prefetch_desc(&p.map_kc);
      tma_prefetch_desc(&p.map_vch);
    }
  }
  // Both CTAs' barriers must exist before either side signals the other.
  cluster_sync();
  const uint32_t q_full_l = mapa_shared(smem_u32(&sm.q_full), 0);
  if (threadIdx.x == 0) {
    // Q does not depend on the mask: start it before the scan.
    if (leader) mbar_arrive_expect_tx(&sm.q_full, 2 * kQBytes);
    tma_load_4d_pair(sQ, &p.map_q, q_full_l, 0, row0, 0, b);
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, 512);
    tmem_relinquish_pair();
  }
  build_codes_x32<kThreads>(ar_b, seg_b, n_key_tok, pad_tokens(n_key_tok), codes, sm.scan,
                            flags0, TileSums{sm.tile_cs_first, sm.tile_cs_last, sm.tile_fast});
  // Warp 0 classifies every key tile for the whole 256-row pair tile (the
  // list must be identical in both CTAs) and compacts the visited ones:
  //   skip    no query of the pair sees any key of the tile
  //   full    every query sees every key (no per-element predicate)
  //   partial per-row visible prefix, FAST hole for expert rows
  const int n_ktiles = (n_key_tok + kBN - 1) / kBN;
  if (warp == 0) {
    int any_e = 0, all_e = 1;
    for (int t = tq0 + lane; t <= tq1; t += 32) {
      const int e = (codes[t] >> 1) & 1;
      any_e |= e;
      all_e &= e;
    }
    any_e = __any_sync(0xffffffffu, any_e);
    all_e = __all_sync(0xffffffffu, all_e);
    const uint32_t csq0 = codes[tq0] >> 2, csq1 = codes[tq1] >> 2;
    int base = 0;
    for (int t0 = 0; t0 < n_ktiles; t0 += 32) {
      const int t = t0 + lane;
      int c = 0;
      bool any_f = false;
      if (t < n_ktiles) {
        const uint32_t csk0 = sm.tile_cs_first[t], csk1 = sm.tile_cs_last[t];
        any_f = (sm.tile_fast[t] & 1) != 0;
        const bool all_f = (sm.tile_fast[t] & 2) != 0;
        const bool complete = (t + 1) * kBN <= n_key_tok;
        if (csk0 > csq1 || (all_e && all_f)) c = 0;
        else if (csk1 <= csq0 && !(any_e && any_f) && complete) c = 1;
        else c = 2;
      }
      const unsigned m = __ballot_sync(0xffffffffu, c != 0);
      if (c != 0) {
        const int pos = base + __popc(m & ((1u << lane) - 1));
        sm.list[pos] = (uint16_t)(t | (c == 2 ? kTilePartial : 0) | (any_f ? kTileAnyFast : 0));
      }
      base += __popc(m);
    }
    if (lane == 0) sm.n_list = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = sm.tmem_base;
  const uint32_t tO = tmem + kColO;
  const uint32_t tS = tmem + kColS;      // S[b] at +128*b

  const int n_total = n_cache + sm.n_list;
  const int per = (n_total + p.n_splits - 1) / p.n_splits;
  const int it_begin = min(split * per, n_total);
  const int it_end = min(it_begin + per, n_total);
  const int n_it = it_end - it_begin;

  if (warp == 0) {
    // ------------------------------------------------- producer (both CTAs)
    if (n_it > 0) {
      uint32_t u = 0;
      auto load = [&](int idx, bool is_v) -> bool {
        const KvTile kt = kv_tile_at<kSuffix>(sm, idx, n_cache, p.P);
        const int s = (int)(u % kStages);
        const uint32_t rel = u / kStages;
        if (rel > 0) {
          const bool ok = wait_or_abort(&sm.kv_empty[s], (rel - 1) & 1, sm, ctl);
          if (!__all_sync(0xffffffffu, ok)) return false;
        }
        if (lane == 0) {
          const uint32_t full_l = mapa_shared(smem_u32(&sm.kv_full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&sm.kv_full[s], 2 * kItemBytes);
          uint8_t* dst = ring + s * kItemBytes;
          if (!is_v) {   // this CTA's 64 keys of the tile, all 256 columns
            const CUtensorMap* map = kt.src ? &p.map_kc : &p.map_k;
            tma_load_4d_pair(dst, map, full_l, 0, kt.tile * kBN + 64 * (int)rank, 0, b);
          } else {       // all 128 keys of the tile, this CTA's 128 columns
            const CUtensorMap* map = kt.src ? &p.map_vch : &p.map_vh;
            tma_load_4d_pair(dst, map, full_l, 0, kt.tile * kBN, 2 * (int)rank, b);
          }
        }
        __syncwarp();
        ++u;
        return true;
      };
      bool ok = true;
      for (int i = it_begin; i < it_end && ok; ++i) {
        ok = load(i, false);
        if (ok && i > it_begin) ok = load(i - 1, true);
      }
      if (ok) ok = load(it_end - 1, true);
      // On failure, loads already issued land on their own (bounded by the TMA);
      // the cluster barrier at the end keeps both CTAs alive until then.
    }
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (even CTA only)
    if (leader && n_it > 0) {
      bool ok = __all_sync(0xffffffffu, wait_or_abort(&sm.q_full, 0, sm, ctl));
      tc_fence_after();
      const uint64_t qdesc0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(ring), 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(smem_u32(ring), kVBlk, 1024);
      auto commit_both = [&](uint64_t* bar) {
        umma_commit_pair(mapa_shared(smem_u32(bar), 0));
        umma_commit_pair(mapa_shared(smem_u32(bar), 1));
      };
      uint32_t u = 0;
      auto pv = [&](int x) -> bool {
        const int bp = x & 1;
        if (!__all_sync(0xffffffffu, wait_or_abort(&sm.p_full[bp], (x >> 1) & 1, sm, ctl)))
          return false;
        const int s = (int)(u % kStages);
        if (!__all_sync(0xffffffffu, wait_or_abort(&sm.kv_full[s], (u / kStages) & 1, sm, ctl)))
          return false;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t vd = vdesc0 + (uint64_t)((s * kItemBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            // B = V[16 keys x (128 columns per CTA)], MN-major: 8-key groups
            // 1024 B apart, 64-column blocks 16 KB apart; a K step is 16 rows.
            umma_pair_ts(tO, tS + 128 * bp + kk * 8, vd + (uint64_t)((kk * 2048) >> 4),
                         kIdescPV, (x > 0 || kk > 0) ? 1u : 0u);
          }
          commit_both(&sm.kv_empty[s]);
          commit_both(&sm.o_done);
        }
        __syncwarp();
        ++u;
        return true;
      };
      for (int i = it_begin; i < it_end && ok; ++i) {
        const int li = i - it_begin;
        const int s = (int)(u % kStages);
        ok = __all_sync(0xffffffffu, wait_or_abort(&sm.kv_full[s], (u / kStages) & 1, sm, ctl));
        if (!ok) break;
        if (li >= 2) {
          // S[li%2] still holds P of tile li-2, the A operand of PV(li-2):
          // this QK may only overwrite it once that PV has finished.
          ok = __all_sync(0xffffffffu, wait_or_abort(&sm.o_done, (li - 2) & 1, sm, ctl));
          if (!ok) break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint64_t kd = kdesc0 + (uint64_t)((s * kItemBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            // A = Q[128 rows per CTA x 16 d], B = K[64 keys per CTA x 16 d],
            // both K-major: 8-row groups 1024 B apart; the K step walks 32 B
            // inside a 64-column block, then the next block.
            const uint32_t qoff = (uint32_t)((kk >> 2) * kQBlk + (kk & 3) * 32);
            const uint32_t koff = (uint32_t)((kk >> 2) * kKBlk + (kk & 3) * 32);
            umma_pair_ss(tS + 128 * (li & 1), qdesc0 + (uint64_t)(qoff >> 4),
                         kd + (uint64_t)(koff >> 4), kIdescQK, kk > 0 ? 1u : 0u);
          }
          commit_both(&sm.kv_empty[s]);
          commit_both(&sm.s_full[li & 1]);
        }
        __syncwarp();
        ++u;
        if (li >= 1) ok = pv(li - 1);
      }
      if (ok) ok = pv(n_it - 1);
      if (lane == 0) umma_commit_pair(smem_u32(&sm.drain));
      __syncwarp();
      (void)mbar_wait(&sm.drain, 0, ctl);
    }
  } else {
    // ------------------------------------ softmax / epilogue (both CTAs)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;             // row of this thread in the CTA
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int tok = min(tq0 + ((int)rank * kBM + r) / p.Hq, tq1);
    const uint32_t cq = codes[tok];
    const uint32_t csq = cq >> 2;
    const bool row_expert = (cq & 2u) != 0;
    const float c = p.scale_log2;                  // > 0
    const uint32_t p_full_l0 = mapa_shared(smem_u32(&sm.p_full[0]), 0);
    const uint32_t p_full_l1 = mapa_shared(smem_u32(&sm.p_full[1]), 0);
    float m_run = -INFINITY;
    float l_run = 0.f;
    bool ok = true;

    for (int i = it_begin; i < it_end && ok; ++i) {
      const int li = i - it_begin;
      const int bs = li & 1;
      if (!wait_or_abort(&sm.s_full[bs], (li >> 1) & 1, sm, ctl)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const KvTile kt = kv_tile_at<kSuffix>(sm, i, n_cache, p.P);
      float x[kBN];
      {
        // all four 32-column loads in flight, one wait
        uint32_t r0[32], r1[32], r2[32], r3[32];
        tmem_ld32(tS + lane_off + 128 * bs, r0);
        tmem_ld32(tS + lane_off + 128 * bs + 32, r1);
        tmem_ld32(tS + lane_off + 128 * bs + 64, r2);
        tmem_ld32(tS + lane_off + 128 * bs + 96, r3);
        tmem_ld_wait();
        reg_fence(r0);
        reg_fence(r1);
        reg_fence(r2);
        reg_fence(r3);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          x[e] = __uint_as_float(r0[e]);
          x[32 + e] = __uint_as_float(r1[e]);
          x[64 + e] = __uint_as_float(r2[e]);
          x[96 + e] = __uint_as_float(r3[e]);
        }
      }
      if (kt.partial) {
        const int k0 = kt.tile * kBN;
        int e;
        bool hole = false;
        if (kSuffix && kt.src == 1) {
          e = min(kBN, p.P - k0);
        } else {
          e = 0;
#pragma unroll
          for (int step = kBN; step >= 1; step >>= 1) {
            const int probe = e + step;
            if (probe <= kBN && (uint32_t)(codes[k0 + probe - 1] >> 2) <= csq) e = probe;
          }
          e = min(e, n_key_tok - k0);
          hole = row_expert && kt.any_fast;
        }
        if (hole) {
          const uint4* kc = reinterpret_cast<const uint4*>(codes + k0);
#pragma unroll
          for (int g = 0; g < kBN / 8; ++g) {
            const uint4 v4 = kc[g];
            const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
            for (int h = 0; h < 8; ++h) {
              const int j = 8 * g + h;
              const bool fast = ((wv[h >> 1] >> (16 * (h & 1))) & 1u) != 0;
              x[j] = (j < e && !fast) ? x[j] : -INFINITY;
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < kBN; ++j) x[j] = j < e ? x[j] : -INFINITY;
        }
      }
      float mt[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) mt[j] = fmaxf(fmaxf(x[j], x[j + 32]), fmaxf(x[j + 64], x[j + 96]));
#pragma unroll
      for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) mt[j] = fmaxf(mt[j], mt[j + w]);
      const float mx = mt[0] * c;

      // Lazy rescaling (exact: O and l always share the reference max).
      const bool upd = mx > m_run + kRescaleThreshold;
      const float m_new = upd ? mx : m_run;
      const float alpha = ex2(m_run - m_new);
      const bool need_o = upd && (m_run != -INFINITY);
      l_run *= (m_run == -INFINITY) ? 0.f : alpha;
      m_run = m_new;
      const float nm = (m_run == -INFINITY) ? 0.f : -m_run;
      float ls[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      uint32_t pk[64];
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const float p0 = ex2(fmaf(x[2 * e], c, nm));
        const float p1 = ex2(fmaf(x[2 * e + 1], c, nm));
        ls[e & 7] += p0 + p1;
        pk[e] = pack_bf16x2_rna(p0, p1);
      }
      l_run += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));

      // No TMEM write of this tile (O rescale or P) may overlap PV of the
      // previous tile: in the CTA-pair form a P store racing the running pair
      // MMA corrupted results.  PV(li-1) has normally finished long before the
      // exponentials above are done, so this wait is free in steady state.
      if (li >= 1) {
        if (!wait_or_abort(&sm.o_done, (li - 1) & 1, sm, ctl)) ok = false;
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, need_o)) {
        const float a = need_o ? alpha : 1.f;
#pragma unroll 1
        for (int cc = 0; cc < kD / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + 32 * cc, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
          tmem_st32(tO + lane_off + 32 * cc, o);
        }
      }
      {
        uint32_t (&pk0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[0]);
        uint32_t (&pk1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[32]);
        tmem_st32(tS + lane_off + 128 * bs, pk0);
        tmem_st32(tS + lane_off + 128 * bs + 32, pk1);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(bs ? p_full_l1 : p_full_l0);
    }

    if (ok && n_it > 0) {
      if (!wait_or_abort(&sm.o_done, (n_it - 1) & 1, sm, ctl)) ok = false;
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && n_it > 0) {
      tc_fence_after();
      const long long grow = (long long)b * rows_per_b + row0 + r;
      const bool row_valid = row0 + r < rows_per_b;
      if (p.n_splits == 1) {
        const float inv = 1.f / l_run;
        // Q is dead once the last PV has finished: stage the bf16 rows there.
        uint8_t* stage = sQ + quarter * 16384;
#pragma unroll 1
        for (int cc = 0; cc < kD / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + 32 * cc, o);
          tmem_ld_wait();
          reg_fence(o);
          uint32_t ob[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            ob[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv,
                                __uint_as_float(o[2 * e + 1]) * inv);
          uint8_t* blk = stage + (cc >> 1) * 4096 + lane * 128;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int unit = (cc & 1) * 4 + q4;
            *reinterpret_cast<uint4*>(blk + ((unit ^ (lane & 7)) << 4)) =
                make_uint4(ob[4 * q4], ob[4 * q4 + 1], ob[4 * q4 + 2], ob[4 * q4 + 3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_4d(&p.map_o, stage, 0, row0 + quarter * 32, 0, b);
          tma_store_commit();
          tma_store_wait_all();
        }
        if (!kSuffix && p.lse && row_valid)
          p.lse[grow] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
      } else {
        // Split-K partial: unnormalised O and (m, l) for the combine kernel.
        // tcgen05.ld is warp-collective (.sync.aligned): every lane loads,
        // only lanes holding a real row store.
        const long long slot = ((long long)split * p.B + b) * rows_per_b + row0 + r;
        float* wo = p.ws + slot * kD;
#pragma unroll 1
        for (int cc = 0; cc < kD / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + 32 * cc, o);
          tmem_ld_wait();
          reg_fence(o);
          if (row_valid) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(wo + 32 * cc + e) =
                  make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                              __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]));
          }
        }
        if (row_valid) {
          float* wml = p.ws + (long long)p.n_splits * p.B * rows_per_b * kD + slot * 2;
          wml[0] = m_run;
          wml[1] = l_run;
        }
      }
    }
    if (n_it == 0 && p.n_splits > 1 && row0 + r < rows_per_b) {
      const long long slot = ((long long)split * p.B + b) * rows_per_b + row0 + r;
      float* wml = p.ws + (long long)p.n_splits * p.B * rows_per_b * kD + slot * 2;
      wml[0] = -INFINITY;
      wml[1] = 0.f;
    }
  }

  // The Q load was issued before the key tiles were counted: a split with no
  // tiles (or one that gave up) must still let both halves land before the
  // CTAs leave.  Completed already in every other case, so this returns at once.
  if (leader && threadIdx.x == 0) (void)mbar_wait(&sm.q_full, 0, ctl);
  // Neither CTA may leave while its partner can still signal its barriers or
  // read its shared memory; then both free their TMEM.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Merges split-K partials: out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s
// with M = max_s m_s (the log-sum-exp rule).  One warp per output row; each
// lane handles 8 of the 256 columns.  HBM-bound: it reads the fp32 partials
// once and writes the bf16 row once.
__global__ void __launch_bounds__(256)
    combine_kernel(const float* __restrict__ ws, __nv_bfloat16* __restrict__ out, int n_splits,
                   long long n_rows) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const float* ml = ws + (long long)n_splits * n_rows * kD;
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, ml[(s * n_rows + row) * 2]);
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float L = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float m = ml[(s * n_rows + row) * 2];
    const float l = ml[(s * n_rows + row) * 2 + 1];
    if (l == 0.f) continue;
    const float w = ex2(m - M);
    L += w * l;
    const float4* src = reinterpret_cast<const float4*>(ws + (s * n_rows + row) * kD + lane * 8);
    const float4 a = src[0], c = src[1];
    acc[0] += w * a.x; acc[1] += w * a.y; acc[2] += w * a.z; acc[3] += w * a.w;
    acc[4] += w * c.x; acc[5] += w * c.y; acc[6] += w * c.z; acc[7] += w * c.w;
  }
  const float inv = 1.f / L;
  uint4 pk;
  pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  pk.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  pk.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(out + row * kD + lane * 8) = pk;
}

size_t pair_smem_bytes(int n_code_tokens) {
  return 1024 /* alignment slack */ + kOffCodes + (size_t)pad_tokens(n_code_tokens) * 2;
}

}  // namespace

cudaError_t launch_tc_pair(const TcParams& p, bool suffix_mode, const DevCtl& ctl,
                           cudaStream_t st) {
  const int rows = p.Sq * p.Hq;
  const int n_pairs = (rows + 2 * kBM - 1) / (2 * kBM);
  dim3 grid(2 * n_pairs * p.n_splits, p.B);
  const size_t smem = pair_smem_bytes(p.Sq);
  static const cudaError_t attr_err = [] {
    const int most = (int)pair_smem_bytes(kMaxTokens);
    cudaError_t a = cudaFuncSetAttribute(tc_pair_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    cudaError_t b = cudaFuncSetAttribute(tc_pair_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    return a != cudaSuccess ? a : b;
  }();
  if (attr_err != cudaSuccess) return attr_err;
  if (suffix_mode) {
    tc_pair_kernel<true><<<grid, kThreads, smem, st>>>(p, ctl);
  } else {
    tc_pair_kernel<false><<<grid, kThreads, smem, st>>>(p, ctl);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.n_splits <= 1) return e;
  const long long n_rows = (long long)p.B * rows;
  combine_kernel<<<(unsigned)((n_rows + 7) / 8), 256, 0, st>>>(
      p.ws, reinterpret_cast<__nv_bfloat16*>(p.out_ptr), p.n_splits, n_rows);
  return cudaGetLastError();
}

int tc_suffix_splits(int B, int Sq, int P, int Hq) {
  // Split the key tiles over several CTA pairs only when the pairs of one
  // split would leave SMs idle: enough splits to fill the SMs once, each
  // keeping at least two key tiles, at most 8.
  static int n_sm = [] {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
  }();
  const int rows = Sq * Hq;
  const int n_ctas = 2 * ((rows + 2 * kBM - 1) / (2 * kBM)) * B;
  const int tiles = (P + kBN - 1) / kBN + (Sq + kBN - 1) / kBN;
  int s = n_sm / max(n_ctas, 1);
  s = min(s, tiles / 2);
  s = min(s, 8);
  return max(s, 1);
}

size_t tc_suffix_workspace_bytes(int B, int Sq, int P, int Hq) {
  const int s = tc_suffix_splits(B, Sq, P, Hq);
  if (s <= 1) return 0;
  const size_t rows = (size_t)B * Sq * Hq;
  return (size_t)s * rows * (kD + 2) * sizeof(float);
}

}  // namespace piattn
